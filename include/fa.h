/*
 * fa.h -- C ABI of the B200 (sm_100a) tiled, IO-aware exact attention library (libfa.so).
 *
 * The operation is exact scaled-dot-product attention
 *     S = scale * Q K^T,  P = softmax(S) row by row,  O = P V,
 * computed tile by tile with an online softmax so that the N x N matrices S
 * and P never reach device memory ("FlashAttention分块计算优化Transformer显存
 * 效率", section 1.1 for the problem and the tiled loop, section 3.2 for the
 * online softmax, section 2.2 for causal block skipping).  The backward pass
 * keeps only O and one statistic per row and recomputes P tile by tile
 * ("图解Flash Attention运算原理", 总结: Recomputation).
 *
 * Conventions shared by every entry point
 *  - Tensors Q, K, V, O, dO, dQ, dK, dV: bf16, shape [B, H, N, d], contiguous
 *    row-major (d fastest), in device memory of the current CUDA device.
 *  - LSE: fp32 [B, H, N]; LSE[b,h,i] = ln sum_j exp(S_ij), the natural-log
 *    logsumexp of row i of the SCALED, masked scores.
 *  - d must be 64 or 128; B, H, N must be positive (a non-positive size is
 *    rejected, as the capacity model of "14. FlashAttention Memory Model"
 *    rejects non-positive sizes); B*H*N must fit in a 32-bit signed int.
 *  - causal != 0 applies the lower-triangular mask: key j is visible to query
 *    i iff j <= i.  Fully masked key tiles are skipped, not computed.
 *  - scale: finite; a value <= 0 selects 1/sqrt(d).
 *  - Every pointer must be non-null and 16-byte aligned.  Outputs must not
 *    overlap inputs or each other.
 *  - stream: a cudaStream_t passed as void* (NULL = the legacy default stream).
 *    Calls are asynchronous: they validate, enqueue and return.  Validation
 *    and launch failures are returned synchronously and nothing is written.
 *    A stall inside a kernel (every internal wait has a wall-clock limit of
 *    2 s) is reported by fa_sync_status as FA_ERR_TIMEOUT.
 *  - Ownership: the caller owns every buffer, including the backward
 *    workspace.  The library allocates no device memory and keeps no state
 *    between calls except per-device attribute caches and the device error
 *    word read by fa_sync_status.
 *  - Device: NVIDIA B200 class (compute capability 10.0, sm_100a) only.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = -1,        /* null pointer, bad size, d not in {64,128}, bad scale, overlap */
  FA_ERR_ALIGNMENT = -2,          /* a pointer is not 16-byte aligned */
  FA_ERR_UNSUPPORTED_DEVICE = -3, /* current device is not sm_100, or a pointer is not device memory */
  FA_ERR_LAUNCH = -4,             /* a CUDA call or kernel launch failed */
  FA_ERR_WORKSPACE = -5,          /* backward workspace missing, misaligned or too small */
  FA_ERR_TIMEOUT = -6,            /* a kernel's internal wait ran out (reported by fa_sync_status) */
  FA_ERR_TOO_LARGE = -7           /* fa_bwd_noalloc: B*H*N exceeds FA_NOALLOC_MAX_ROWS */
} fa_status;

/*
 * Forward pass.
 * In:  Q, K, V [B,H,N,d] bf16.
 * Out: O [B,H,N,d] bf16 (O = P V, rounded to nearest even), LSE [B,H,N] fp32.
 * One persistent kernel launch on `stream`: CTA pairs (fa_fwd_2sm_kernel) for
 * d = 128 without the mask, one SM per CTA (fa_fwd_kernel) otherwise.  With
 * the mask the launch carries each CTA's (the paired kernel: each CTA pair's)
 * list of query-tile pairs, computed on the host at the first call for a
 * shape and kept (a few shapes at a time).  Two
 * environment variables, read at each call, select other forms for
 * comparisons: FA_FWD_PAIR=0 / =1 forces the one-SM / paired kernel for
 * d = 128; FA_FWD_BN=64 runs the one-SM kernel with 64-key K/V tiles instead
 * of 128.  FA_FWD_RESCALE=t (0 .. 30, default 8) sets the online-softmax
 * rescale threshold: O is rescaled only when a row maximum grows by more than
 * a factor 2^t.  All forms compute the same O and LSE up to rounding.
 * Returns FA_OK or an fa_status error code (nothing written on error).
 */
int fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int N, int d,
           int causal, float scale, void* stream);

/*
 * Bytes of device workspace fa_bwd needs for these sizes: the fp32 row vector
 * D = rowsum(dO * O) ([B,H,N], rounded up to 256 bytes) followed by the fp32
 * dQ accumulator ([B,H,N,d]).  Enough for fa_bwd_deterministic too, which
 * uses only the D part.  Returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward pass for the loss L = sum(dO * O).
 * In:  Q, K, V, O (the forward's output), dO [B,H,N,d] bf16; LSE [B,H,N] fp32
 *      from fa_fwd with the same causal flag and scale.
 * Out: dQ, dK, dV [B,H,N,d] bf16.
 * Workspace: caller-owned device buffer of at least fa_bwd_workspace_bytes()
 *      bytes, 16-byte aligned, not overlapping any other argument; its
 *      contents on entry do not matter.
 * Three launches, in order on `stream`: the D = rowsum(dO * O) pass (which
 * also zeroes the dQ accumulator); fa_bwd_fused_kernel, persistent (one CTA
 * per SM walking units of 128 keys of a head; with the mask each CTA's list
 * of units is computed on the host at the first call for a shape and kept),
 * which recomputes P = exp(S - LSE) tile by tile and forms all
 * five products of the gradient -- S, dP, dV, dK and the tile's share of dQ,
 * added into the fp32 accumulator by the bulk-copy engine; and a pass that
 * writes dQ = bf16(scale * accumulator).  dK and dV are accumulated in a
 * fixed order and are deterministic; the partial sums of dQ arrive in an
 * order that varies from run to run, so dQ can differ in its last bits
 * between runs (fa_bwd_deterministic does not).
 */
int fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
           void* dQ, void* dK, void* dV, int B, int H, int N, int d, int causal, float scale,
           void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd with bit-reproducible results: the same arguments and outputs, but
 * dQ gets its own kernel (one CTA per 128 query rows) that recomputes S and
 * dP instead of adding partial sums, so every output is written once by one
 * CTA and repeated calls give identical bits.  It performs seven tensor-core
 * products per tile pair instead of five and is slower.  Launches: the D
 * pass, fa_bwd_dkdv_kernel, fa_bwd_dq_kernel.  The workspace must hold at
 * least the D part (4 * B*H*N bytes rounded up to 256); a buffer of
 * fa_bwd_workspace_bytes() always suffices.
 */
int fa_bwd_deterministic(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                         const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int N, int d, int causal,
                         float scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward and backward from host memory to host memory, for callers whose
 * data lives on the host: the pages' problem statement run end to end, with
 * the PCIe copies overlapped with the kernels.
 * In (host or device memory, page-locked host memory for the copies to
 * overlap): Q, K, V, dO [B,H,N,d] bf16.
 * Out (same kinds of memory): O [B,H,N,d] bf16, LSE [B,H,N] fp32, dQ, dK, dV
 * [B,H,N,d] bf16 -- what fa_fwd followed by fa_bwd produce.
 * The B*H heads go in `groups` (1 .. B*H; more are clamped) consecutive groups
 * of ceil(B*H / groups) heads.  Three of the library's own streams, created at
 * the first call on each device and kept, carry the copies of group c to the
 * device, fa_fwd + fa_bwd on group c-1 and the copies of group c-2 back, so
 * both copy directions and the kernels run at the same time.
 * workspace: caller-owned device memory of at least
 * fa_fwd_bwd_host_workspace_bytes(B, H, N, d, groups) bytes (three slots, each
 * holding one group's inputs, outputs and backward workspace), 16-byte
 * aligned.  The call allocates nothing.
 * stream: the pipeline starts after the work already queued on `stream`, and
 * `stream` waits for the whole pipeline: once it synchronizes, the outputs
 * are in host memory.  Calls from several threads are queued one after
 * another.  Returns FA_OK or an fa_status code; validation errors return
 * before anything is queued; an error from a group's kernels returns with
 * earlier groups already queued (outputs then undefined).
 */
size_t fa_fwd_bwd_host_workspace_bytes(int B, int H, int N, int d, int groups);
int fa_fwd_bwd_host(const void* Q, const void* K, const void* V, const void* dO, void* O, float* LSE, void* dQ,
                    void* dK, void* dV, int B, int H, int N, int d, int causal, float scale, int groups,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd for callers that cannot allocate device memory -- for example a
 * plugin whose host runtime hands it only its input and output buffers, or
 * code running under a memory pool that must not grow.  The paper has no
 * counterpart to this entry point.
 *
 * Same arguments, semantics and outputs as fa_bwd_deterministic (the form
 * whose only scratch is the D vector), minus the workspace: the
 * D = rowsum(dO * O) vector lives in a fixed array inside the library
 * (FA_NOALLOC_MAX_ROWS fp32 entries = 4 MiB, held on every GPU that loads the
 * library until the process exits).  The call itself allocates nothing.
 * Results are bit-identical to fa_bwd_deterministic's.
 *  - Sizes: B*H*N must not exceed FA_NOALLOC_MAX_ROWS, else FA_ERR_TOO_LARGE
 *    (nothing is launched).
 *  - Set-up: the first call on each device looks up the array's device address
 *    (with that device current); make that first call before any stream
 *    capture.  The address is remembered per device together with the CUDA
 *    context it belongs to; after a device reset (a new primary context) the
 *    next call looks it up again.
 *  - The array is shared by every call on a device and keeps the last call's
 *    contents; each call overwrites the part it uses before reading it.  Calls
 *    that overlap on the GPU (different streams, no ordering between them) race
 *    on the array: order them or use fa_bwd with separate workspaces.
 */
#define FA_NOALLOC_MAX_ROWS (1 << 20)
int fa_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                   void* dQ, void* dK, void* dV, int B, int H, int N, int d, int causal, float scale,
                   void* stream);

/*
 * Synchronises `stream`, then reports: FA_ERR_LAUNCH if a CUDA error is
 * pending, FA_ERR_TIMEOUT if a kernel of this library recorded a wait
 * timeout since the last call (the record is then cleared), else FA_OK.
 */
int fa_sync_status(void* stream);

/*
 * The raw device error word recorded with the last FA_ERR_TIMEOUT reported
 * by fa_sync_status ((wait site << 8) | code; 0 if none).  For diagnosis.
 */
unsigned int fa_last_error_word(void);

/*
 * The cause of the last FA_ERR_LAUNCH returned by this library, for
 * diagnosis: a cudaError_t value, or 100000 + the CUresult of a failed
 * tensor-map encode (0 if none).
 */
int fa_last_cuda_error(void);

/*
 * Optional per-kernel timing of the backward (profiling aid).  When set,
 * fa_bwd, fa_bwd_deterministic and fa_bwd_noalloc record the four
 * cudaEvent_t handles (passed as void*) on their stream: e0 before the D
 * pass, e1 before the second launch (fa_bwd_fused_kernel, or
 * fa_bwd_dkdv_kernel for the deterministic form), e2 before the third (the
 * dQ conversion, or fa_bwd_dq_kernel), e3 after it.  Events belong to the
 * caller and must stay valid while set; pass four NULLs to stop.  The setting
 * is process-wide.
 */
void fa_bwd_set_phase_events(void* e0, void* e1, void* e2, void* e3);

/*
 * Standard (unfused) attention forward: the comparison column of the HBM
 * access table in "FlashAttention分块计算优化Transformer显存效率", section 2.1
 * (内存访问模式对比).  Computes the same O and LSE as fa_fwd, but writes the
 * score matrix S = scale * Q K^T (fp16) to HBM, reads it back for a row
 * softmax that writes P (bf16) over it, and reads P for O = P V.  Exists to
 * measure the HBM traffic the tiled kernels avoid; every score is computed
 * (the causal mask is applied in the softmax).
 *
 * Arguments as fa_fwd, plus `workspace`: caller-owned device memory of at
 * least fa_fwd_unfused_workspace_bytes(B, H, N, d) bytes, 16-byte aligned,
 * not overlapping any other argument; it holds S, then P, as [B*H][Nr][Nr]
 * 16-bit elements, Nr = N rounded up to a multiple of 128.  Returns
 * FA_ERR_WORKSPACE when it is missing, too small, misaligned or overlaps
 * another argument, otherwise the same codes as fa_fwd.  Asynchronous on `stream`.  The 16-bit S limits LSE accuracy to
 * about max|score| * 2^-11 (it is exact to 1e-3 for scores of magnitude < 2).
 */
size_t fa_fwd_unfused_workspace_bytes(int B, int H, int N, int d);
int fa_fwd_unfused(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int N, int d,
                   int causal, float scale, void* workspace, size_t workspace_bytes, void* stream);

/* Human-readable name of an fa_status value (static string). */
const char* fa_status_string(int status);

/*
 * Name of the kernel fa_fwd launches on the current device for head size d
 * and the given mask flag: "fa_fwd_2sm_kernel" (CTA pairs, d = 128 without
 * the mask) or "fa_fwd_kernel", following FA_FWD_PAIR and FA_FWD_BN as
 * fa_fwd does.  NULL when d is not 64 or 128 or
 * the device is not usable.  Static string, owned by the library.  For
 * labelling timings and profiles; the paper has no counterpart.
 */
const char* fa_fwd_kernel_name(int d, int causal);

/*
 * Name of the kernel that computes dK and dV in fa_bwd for head size d:
 * "fa_bwd_fused_kernel" (which also forms the dQ partial sums).
 * fa_bwd_deterministic runs "fa_bwd_dkdv_kernel" instead.  NULL when d is
 * not 64 or 128.  Static string, owned by the library.  For labelling
 * timings and profiles; the paper has no counterpart.
 */
const char* fa_bwd_dkdv_kernel_name(int d);

/*
 * The per-CTA unit lists the causal kernels follow, for inspection and tests
 * (host only: no GPU, no device call).  kind 0: the causal forward's lists
 * (grid = CTAs of the one-SM kernel, or CTA pairs of the paired kernel)
 * (units = pairs of 128-row query tiles of a head; unit index r*B*H + bh is
 * query-tile pair NP-1-r of head bh, NP = ceil(ceil(N/128)/2)), built for
 * 128-key tiles; kind 1: the persistent fused backward's lists (units = 128-key
 * tiles of a head, numbered in the kernel's grouped longest-first order).
 * Lists hold each unit once: CTA c runs order[start[c] .. start[c+1]).
 * `grid` CTAs (1 .. 160); `start` has room for grid + 1 entries, `order` for
 * max_units.  Returns the number of units (the lists are written), 0 when the
 * shape has no lists (more than 4096 units: the kernels deal the units in
 * serpentine order instead; nothing is written), or FA_ERR_INVALID_ARG (bad
 * kind, sizes or grid, or max_units too small).  The paper has no
 * counterpart: this is how the kernels balance the causal mask's unequal
 * units over the SMs.
 */
int fa_unit_lists(int kind, int B, int H, int N, int d, int grid, unsigned short* start, unsigned short* order,
                  int max_units);

/*
 * Fault-detection self test.  Launches one tiny kernel that waits on a
 * barrier nothing ever signals, with a wall-clock limit of `limit_us`
 * microseconds (1 .. 10,000,000).  The wait runs out, the kernel records
 * FA_ERR_TIMEOUT and returns; the next fa_sync_status(stream) reports it and
 * the CUDA context stays usable.  Nothing faults or traps.
 */
int fa_selftest_wait_timeout(unsigned int limit_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
