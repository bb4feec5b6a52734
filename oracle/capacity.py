"""Capacity model of a materialised score tensor (test infrastructure).

Follows "14. FlashAttention Memory Model", Q1 small check: the bytes of a
materialised score tensor are batch * heads * seq_len^2 * dtype_bytes, and a
non-positive argument is rejected with ValueError.  Used only to check the
statement that the long-sequence workload's S would take 8 GiB in bf16.
"""


def attention_score_bytes(seq_len: int, batch_size: int = 1, num_heads: int = 1,
                          dtype_bytes: int = 2) -> int:
    for value in (seq_len, batch_size, num_heads, dtype_bytes):
        if value <= 0:
            raise ValueError("sizes must be positive")
    return batch_size * num_heads * seq_len * seq_len * dtype_bytes
