// fa_api.cu -- the C ABI of libfa.so: argument validation, TMA descriptor
// encoding and kernel launches for the sm_100a attention kernels.
#include <math.h>
#include <algorithm>
#include <mutex>
#include <queue>
#include <utility>
#include <vector>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_bwd_fused.cuh"
#include "fa_fwd.cuh"
#include "fa_fwd2.cuh"
#include "fa_unfused.cuh"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D view [BH][N][d] of a bf16 [B,H,N,d] tensor; box = 64 columns x box_rows
// rows x 1 head, 128-byte swizzle.  Rows past N read as zero within the head.
int g_last_encode_error = 0;  // CUresult of the last failed tensor-map encode (diagnosis)

bool encode_map(CUtensorMap* m, const void* base, int BH, int N, int d, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    g_last_encode_error = -1;
    return false;
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) g_last_encode_error = static_cast<int>(r);
  return r == CUDA_SUCCESS;
}

// Encoded tensor maps, remembered by (address, heads, rows, head size, box
// rows): a map holds only the address and the layout, so a later call on the
// same tensor -- or on a new tensor of the same shape at the same address --
// reuses it instead of encoding it again.  A small table, replaced round-robin.
struct MapEntry {
  const void* base = nullptr;
  int BH = 0, N = 0, d = 0, box_rows = 0;
  CUtensorMap map;
};
constexpr int kMapCache = 64;
MapEntry g_maps[kMapCache];
int g_maps_next = 0;
std::mutex g_maps_mu;

bool make_map(CUtensorMap* m, const void* base, int BH, int N, int d, int box_rows) {
  {
    std::lock_guard<std::mutex> lock(g_maps_mu);
    for (const MapEntry& e : g_maps)
      if (e.base == base && e.BH == BH && e.N == N && e.d == d && e.box_rows == box_rows) {
        *m = e.map;
        return true;
      }
  }
  if (!encode_map(m, base, BH, N, d, box_rows)) return false;
  std::lock_guard<std::mutex> lock(g_maps_mu);
  MapEntry& e = g_maps[g_maps_next];
  g_maps_next = (g_maps_next + 1) % kMapCache;
  e.base = base;
  e.BH = BH;
  e.N = N;
  e.d = d;
  e.box_rows = box_rows;
  e.map = *m;
  return true;
}

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int checked = 0;  // 0 unknown, 1 supported, -1 unsupported
  int sms = 0;
  int pair_clusters[2] = {0, 0};  // co-resident 2-CTA clusters of the paired forward kernel (non-causal, causal)
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

template <typename Kern>
bool set_smem(Kern k, int bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

// Returns FA_OK and the SM count if the current device is sm_100 and the
// kernels' shared-memory limits are set on it.
int device_ready(int* sms, int* pair_clusters = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_UNSUPPORTED_DEVICE;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED_DEVICE;
  // Binds the device's primary context to this thread (a thread that only had
  // its device set, e.g. an autograd worker, may have none yet); the tensor-map
  // encoder is a driver call and needs it.
  if (cudaSetDevice(dev) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_UNSUPPORTED_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (di.checked == 0) {
    int major = 0, minor = 0, n = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    bool ok = (major == 10 && minor == 0) && n > 0;
    ok = ok && set_smem(fa::fa_fwd_kernel<64, false>, fa::FwdCfg<64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_fwd_kernel<64, true>, fa::FwdCfg<64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_fwd_kernel<128, false>, fa::FwdCfg<128>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_fwd_kernel<128, true>, fa::FwdCfg<128>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_fwd_kernel<64, false, 64>, fa::FwdCfg<64, 64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_fwd_kernel<64, true, 64>, fa::FwdCfg<64, 64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_fwd_kernel<128, false, 64>, fa::FwdCfg<128, 64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_fwd_kernel<128, true, 64>, fa::FwdCfg<128, 64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_bwd_dkdv_kernel<64, false>, fa::DkdvCfg<64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_bwd_dkdv_kernel<64, true>, fa::DkdvCfg<64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_bwd_dkdv_kernel<128, false>, fa::DkdvCfg<128>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_bwd_dkdv_kernel<128, true>, fa::DkdvCfg<128>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_bwd_dq_kernel<64, false>, fa::DqCfg<64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_bwd_dq_kernel<64, true>, fa::DqCfg<64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_bwd_dq_kernel<128, false>, fa::DqCfg<128>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_bwd_dq_kernel<128, true>, fa::DqCfg<128>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_fwd_2sm_kernel<false>, fa::Fwd2Cfg::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_fwd_2sm_kernel<true>, fa::Fwd2Cfg::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_bwd_fused_kernel<64, false>, fa::FusedCfg<64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_bwd_fused_kernel<64, true>, fa::FusedCfg<64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_bwd_fused_kernel<128, false>, fa::FusedCfg<128>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_bwd_fused_kernel<128, true>, fa::FusedCfg<128>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_unf_scores_kernel<64>, fa::UnfScoresCfg<64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_unf_scores_kernel<128>, fa::UnfScoresCfg<128>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_unf_pv_kernel<64>, fa::UnfPvCfg<64>::SMEM_BYTES);
    ok = ok && set_smem(fa::fa_unf_pv_kernel<128>, fa::UnfPvCfg<128>::SMEM_BYTES);
    for (int c = 0; c < 2 && ok; ++c) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * n, 1, 1);
      cfg.blockDim = dim3(fa::Fwd2Cfg::THREADS, 1, 1);
      cfg.dynamicSmemBytes = fa::Fwd2Cfg::SMEM_BYTES;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      const cudaError_t e = c ? cudaOccupancyMaxActiveClusters(&clusters, fa::fa_fwd_2sm_kernel<true>, &cfg)
                              : cudaOccupancyMaxActiveClusters(&clusters, fa::fa_fwd_2sm_kernel<false>, &cfg);
      di.pair_clusters[c] = (e == cudaSuccess) ? clusters : 0;
    }
    cudaGetLastError();
    di.checked = ok ? 1 : -1;
    di.sms = n;
  }
  if (di.checked != 1) return FA_ERR_UNSUPPORTED_DEVICE;
  *sms = di.sms;
  if (pair_clusters) {
    pair_clusters[0] = di.pair_clusters[0];
    pair_clusters[1] = di.pair_clusters[1];
  }
  return FA_OK;
}

cudaEvent_t g_phase_events[4] = {nullptr, nullptr, nullptr, nullptr};
int g_last_cuda_error = 0;

// Status of the launches just made.  Errors left pending by earlier, unrelated
// runtime calls on this thread are cleared before launching (see
// clear_stale_error), so an error seen here belongs to these launches.
int launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return FA_OK;
  g_last_cuda_error = static_cast<int>(e);
  return FA_ERR_LAUNCH;
}
void clear_stale_error() { (void)cudaGetLastError(); }

// A tensor-map encode failed: reported as FA_ERR_LAUNCH with
// fa_last_cuda_error() = 100000 + the driver's CUresult (or 99999 if the
// driver entry point could not be found).
int encode_failed() {
  g_last_cuda_error = 100000 + g_last_encode_error;
  return FA_ERR_LAUNCH;
}
std::mutex g_events_mu;

// Device-memory allocations already seen, as address ranges per device: a
// pointer inside one of them is device memory of that device without asking
// the driver again (the check costs a driver call per pointer otherwise).
// Ranges come from cuMemGetAddressRange on pointers the runtime reported as
// device memory of the current device.  Freeing an allocation does not
// remove its range; the addresses of freed device memory are only handed out
// again for device memory.
struct RangeEntry {
  uintptr_t lo = 0, hi = 0;
  int dev = -1;
};
constexpr int kRangeCache = 64;
RangeEntry g_ranges[kRangeCache];
int g_ranges_next = 0;
std::mutex g_ranges_mu;

using GetAddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
GetAddressRangeFn address_range_fn() {
  static GetAddressRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetAddressRangeFn>(p);
  });
  return fn;
}

// True if [p, p + bytes) is device (or managed) memory of the current device.
bool is_device_ptr(const void* p, size_t bytes = 1) {
  int dev = 0;
  cudaGetDevice(&dev);
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p), hi = lo + (bytes ? bytes : 1);
  {
    std::lock_guard<std::mutex> lock(g_ranges_mu);
    for (int i = 1; i <= kRangeCache; ++i) {  // most recently added first
      const RangeEntry& e = g_ranges[(g_ranges_next - i + kRangeCache) % kRangeCache];
      if (e.dev == dev && lo >= e.lo && hi <= e.hi) return true;
    }
  }
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (!((a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) && a.device == dev)) return false;
  CUdeviceptr base = 0;
  size_t size = 0;
  GetAddressRangeFn fn = address_range_fn();
  if (fn && fn(&base, &size, static_cast<CUdeviceptr>(lo)) == CUDA_SUCCESS && size > 0) {
    std::lock_guard<std::mutex> lock(g_ranges_mu);
    RangeEntry& e = g_ranges[g_ranges_next];
    g_ranges_next = (g_ranges_next + 1) % kRangeCache;
    e.lo = static_cast<uintptr_t>(base);
    e.hi = static_cast<uintptr_t>(base) + size;
    e.dev = dev;
  }
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;
};
bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

int check_sizes(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(B) * H * N;
  if (rows > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

float effective_scale(float scale, int d, bool* ok) {
  *ok = isfinite(scale);
  return scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(d));
}

// Unit lists of the causal one-SM forward.  A unit is a pair of 128-row query
// tiles of one head; pair p of a head runs (2p+1) + (2p+2) key-tile steps
// (scaled by 128 / BN), plus about one step per query tile of fixed cost.
// Order: heads in groups whose K and V fit in 32 MiB of L2, inside a group the
// longest units first; then a longest-processing-time assignment: each unit
// in that order goes to the CTA with the least work so far.  Each CTA runs its
// units in assignment order.  Lists are cached per shape (they depend only on
// the head count, N, d, the key tile and the grid).
struct UnitListEntry {
  int BH = -1, N = 0, d = 0, bn = 0, grid = 0;
  fa::FwdUnitList list;
};
constexpr int kListCache = 4;
UnitListEntry g_lists[kListCache];
int g_lists_next = 0;
std::mutex g_lists_mu;

constexpr long long kFwdGroupBytes = 32ll << 20;  // K and V of a head group

// Longest-processing-time assignment of units, taken in the given order (the
// caller puts the longest first), each to the CTA with the least work so far;
// each CTA runs its units in assignment order.
void lpt_assign(fa::UnitList* L, const std::vector<int>& order, const std::vector<long long>& cost, int grid) {
  using Load = std::pair<long long, int>;  // (work so far, CTA): the smallest on top
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int c = 0; c < grid; ++c) heap.push({0, c});
  std::vector<int> owner(order.size()), count(grid, 0);
  for (size_t i = 0; i < order.size(); ++i) {
    Load top = heap.top();
    heap.pop();
    owner[i] = top.second;
    ++count[top.second];
    heap.push({top.first + cost[i], top.second});
  }
  L->n = static_cast<int>(order.size());
  L->start[0] = 0;
  for (int c = 0; c < grid; ++c) L->start[c + 1] = static_cast<unsigned short>(L->start[c] + count[c]);
  std::vector<int> fill(L->start, L->start + grid);
  for (size_t i = 0; i < order.size(); ++i) L->order[fill[owner[i]]++] = static_cast<unsigned short>(order[i]);
}

bool build_unit_list(fa::FwdUnitList* L, int BH, int N, int d, int bn, int grid) {
  const int NKT = (N + bn - 1) / bn, NQT = (N + 127) / 128, NP = (NQT + 1) / 2, R = 128 / bn;
  const long long units = static_cast<long long>(BH) * NP;
  if (units > fa::FwdUnitList::kMaxUnits || grid > fa::FwdUnitList::kMaxCtas || grid < 1) return false;
  const long long per_head = 4ll * N * d;  // K and V, bf16
  long long g = kFwdGroupBytes / per_head;
  const int G = g >= BH ? BH : (g < 1 ? 1 : static_cast<int>(g));
  std::vector<int> order;
  order.reserve(units);
  for (int g0 = 0; g0 < BH; g0 += G)
    for (int r = 0; r < NP; ++r)
      for (int bh = g0; bh < BH && bh < g0 + G; ++bh) order.push_back(r * BH + bh);
  std::vector<long long> cost(order.size());
  for (size_t i = 0; i < order.size(); ++i) {
    const int qp = NP - 1 - order[i] / BH;
    const int nk0 = std::min((2 * qp + 1) * R, NKT), nk1 = std::min((2 * qp + 2) * R, NKT);
    cost[i] = nk0 + nk1 + 2 * R;
  }
  lpt_assign(L, order, cost, grid);
  return true;
}

// The list for a causal launch, copied into *out; false: use the serpentine deal.
bool causal_unit_list(fa::FwdUnitList* out, int BH, int N, int d, int bn, int grid) {
  std::lock_guard<std::mutex> lock(g_lists_mu);
  for (const UnitListEntry& e : g_lists)
    if (e.BH == BH && e.N == N && e.d == d && e.bn == bn && e.grid == grid) {
      *out = e.list;
      return e.list.n > 0;
    }
  UnitListEntry& e = g_lists[g_lists_next];
  g_lists_next = (g_lists_next + 1) % kListCache;
  e.BH = BH, e.N = N, e.d = d, e.bn = bn, e.grid = grid;
  if (!build_unit_list(&e.list, BH, N, d, bn, grid)) e.list.n = 0;
  *out = e.list;
  return e.list.n > 0;
}

// Unit lists of the persistent fused backward with the mask.  Unit u is key
// tile kt of head bh in the kernel's grouped order (heads in groups whose K
// and V fit in 32 MiB of L2, the first key tiles -- those that see the most
// query tiles -- first); its cost is its query tiles plus one for the unit's
// fixed work (K and V loads, the dK and dV stores, mostly overlapped).
UnitListEntry g_bwd_lists[kListCache];
int g_bwd_lists_next = 0;

bool build_bwd_unit_list(fa::UnitList* L, int BH, int N, int d, int grid) {
  const int NKT = (N + 127) / 128, NQT = (N + 63) / 64;
  const long long units = static_cast<long long>(BH) * NKT;
  if (units > fa::UnitList::kMaxUnits || grid > fa::UnitList::kMaxCtas || grid < 1) return false;
  const int G = fa::causal_head_group(BH, N, d);
  std::vector<int> order(units);
  std::vector<long long> cost(units);
  for (int u = 0; u < units; ++u) {
    int bh, kt;
    fa::causal_grouped_unit(u, BH, NKT, G, bh, kt);
    order[u] = u;
    cost[u] = (NQT - (kt * 128) / 64) + 1;
  }
  lpt_assign(L, order, cost, grid);
  return true;
}

bool causal_bwd_unit_list(fa::UnitList* out, int BH, int N, int d, int grid) {
  std::lock_guard<std::mutex> lock(g_lists_mu);
  for (const UnitListEntry& e : g_bwd_lists)
    if (e.BH == BH && e.N == N && e.d == d && e.grid == grid) {
      *out = e.list;
      return e.list.n > 0;
    }
  UnitListEntry& e = g_bwd_lists[g_bwd_lists_next];
  g_bwd_lists_next = (g_bwd_lists_next + 1) % kListCache;
  e.BH = BH, e.N = N, e.d = d, e.bn = 128, e.grid = grid;
  if (!build_bwd_unit_list(&e.list, BH, N, d, grid)) e.list.n = 0;
  *out = e.list;
  return e.list.n > 0;
}

}  // namespace

extern "C" {

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_ALIGNMENT: return "FA_ERR_ALIGNMENT";
    case FA_ERR_UNSUPPORTED_DEVICE: return "FA_ERR_UNSUPPORTED_DEVICE";
    case FA_ERR_LAUNCH: return "FA_ERR_LAUNCH";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_TOO_LARGE: return "FA_ERR_TOO_LARGE";
    default: return "FA_ERR_UNKNOWN";
  }
}

// d = 128 non-causal: the paired (2-SM) kernel (faster there); causal and
// d = 64 run the 1-SM kernel.  FA_FWD_PAIR=0 / =1 forces one or the other for
// d = 128 (comparisons and tests).  `clusters`: CTA pairs that fit at once.
// Keys per K/V tile of the one-SM kernel: 128, or 64 when FA_FWD_BN=64
// (tile-size comparisons; 64-key tiles also rule out the paired kernel).
static int fwd_key_tile() {
  const char* bn_env = getenv("FA_FWD_BN");
  return (bn_env && strcmp(bn_env, "64") == 0) ? 64 : 128;
}

// Online-softmax rescale threshold in log2 units: O is rescaled only when a
// row max grows by more than 2^threshold.  FA_FWD_RESCALE (0 .. 30) overrides
// the default 8; 0 rescales on every growth.  Any value gives the same result
// up to rounding: P stays below 2^threshold, far inside fp32 and bf16 range.
static float fwd_rescale_log2() {
  const char* env = getenv("FA_FWD_RESCALE");
  if (!env) return 8.f;
  char* end = nullptr;
  const float v = strtof(env, &end);
  return (end != env && v >= 0.f && v <= 30.f) ? v : 8.f;
}

static bool fwd_use_pair(int d, int causal, int clusters) {
  const char* pair_env = getenv("FA_FWD_PAIR");
  bool use_pair = d == 128 && clusters > 0 && !causal;
  if (pair_env && strcmp(pair_env, "0") == 0) use_pair = false;
  if (pair_env && strcmp(pair_env, "1") == 0) use_pair = d == 128 && clusters > 0;
  return use_pair && fwd_key_tile() == 128;
}

const char* fa_fwd_kernel_name(int d, int causal) {
  if (d != 64 && d != 128) return nullptr;
  int sms = 0, pair_clusters[2] = {0, 0};
  if (device_ready(&sms, pair_clusters)) return nullptr;
  return fwd_use_pair(d, causal, pair_clusters[causal ? 1 : 0]) ? "fa_fwd_2sm_kernel" : "fa_fwd_kernel";
}

int fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int N, int d,
           int causal, float scale, void* stream) {
  int rc = check_sizes(B, H, N, d);
  if (rc) return rc;
  if (!Q || !K || !V || !O || !LSE) return FA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE)) return FA_ERR_ALIGNMENT;
  bool scale_ok = false;
  const float sc = effective_scale(scale, d, &scale_ok);
  if (!scale_ok) return FA_ERR_INVALID_ARG;
  const size_t tbytes = static_cast<size_t>(B) * H * N * d * 2, lbytes = static_cast<size_t>(B) * H * N * 4;
  const Range rq{(uintptr_t)Q, (uintptr_t)Q + tbytes}, rk{(uintptr_t)K, (uintptr_t)K + tbytes},
      rv{(uintptr_t)V, (uintptr_t)V + tbytes}, ro{(uintptr_t)O, (uintptr_t)O + tbytes},
      rl{(uintptr_t)LSE, (uintptr_t)LSE + lbytes};
  if (overlaps(ro, rq) || overlaps(ro, rk) || overlaps(ro, rv) || overlaps(ro, rl) || overlaps(rl, rq) ||
      overlaps(rl, rk) || overlaps(rl, rv))
    return FA_ERR_INVALID_ARG;
  int sms = 0, pair_clusters[2] = {0, 0};
  if ((rc = device_ready(&sms, pair_clusters))) return rc;
  if (!is_device_ptr(Q, tbytes) || !is_device_ptr(K, tbytes) || !is_device_ptr(V, tbytes) ||
      !is_device_ptr(O, tbytes) || !is_device_ptr(LSE, lbytes))
    return FA_ERR_UNSUPPORTED_DEVICE;
  const int BH = B * H;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, BH, N, d, 128) || !make_map(&mk, K, BH, N, d, 128) || !make_map(&mv, V, BH, N, d, 128))
    return encode_failed();
  clear_stale_error();
  const float rescale = fwd_rescale_log2();
  const int clusters = pair_clusters[causal ? 1 : 0];
  if (fwd_use_pair(d, causal, clusters)) {
    CUtensorMap mkh;
    if (!make_map(&mkh, K, BH, N, d, 64)) return encode_failed();
    const int nqp = (N + 255) / 256, punits = BH * nqp;
    const int pairs = punits < clusters ? punits : clusters;
    const float sl2p = sc * fa::kLog2e;
    cudaStream_t sp = static_cast<cudaStream_t>(stream);
    auto* op = static_cast<__nv_bfloat16*>(O);
    if (causal) {
      fa::FwdUnitList pl;  // per CTA pair (n = 0: serpentine deal)
      pl.n = 0;
      causal_unit_list(&pl, BH, N, d, 128, pairs);
      fa::fa_fwd_2sm_kernel<true><<<2 * pairs, fa::Fwd2Cfg::THREADS, fa::Fwd2Cfg::SMEM_BYTES, sp>>>(mq, mkh, mv, op, LSE, BH, N, sl2p, rescale, pl);
    } else {
      fa::fa_fwd_2sm_kernel<false><<<2 * pairs, fa::Fwd2Cfg::THREADS, fa::Fwd2Cfg::SMEM_BYTES, sp>>>(mq, mkh, mv, op, LSE, BH, N, sl2p, rescale, fa::FwdNoList{0});
    }
    return launch_status();
  }
  const int nqt = (N + 127) / 128, units = BH * ((nqt + 1) / 2);
  const int grid = units < sms ? units : sms;
  const float sl2 = sc * fa::kLog2e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* o = static_cast<__nv_bfloat16*>(O);
  fa::FwdUnitList ul;  // causal: this shape's unit lists (n = 0: serpentine deal)
  ul.n = 0;
  if (causal) causal_unit_list(&ul, BH, N, d, fwd_key_tile(), grid);
  if (fwd_key_tile() == 64) {  // 64-key tiles: for tile-size comparisons only
    CUtensorMap mk64, mv64;
    if (!make_map(&mk64, K, BH, N, d, 64) || !make_map(&mv64, V, BH, N, d, 64)) return encode_failed();
    if (d == 64) {
      if (causal) fa::fa_fwd_kernel<64, true, 64><<<grid, fa::FwdCfg<64, 64>::THREADS, fa::FwdCfg<64, 64>::SMEM_BYTES, s>>>(mq, mk64, mv64, o, LSE, BH, N, sl2, rescale, ul);
      else fa::fa_fwd_kernel<64, false, 64><<<grid, fa::FwdCfg<64, 64>::THREADS, fa::FwdCfg<64, 64>::SMEM_BYTES, s>>>(mq, mk64, mv64, o, LSE, BH, N, sl2, rescale, fa::FwdNoList{0});
    } else {
      if (causal) fa::fa_fwd_kernel<128, true, 64><<<grid, fa::FwdCfg<128, 64>::THREADS, fa::FwdCfg<128, 64>::SMEM_BYTES, s>>>(mq, mk64, mv64, o, LSE, BH, N, sl2, rescale, ul);
      else fa::fa_fwd_kernel<128, false, 64><<<grid, fa::FwdCfg<128, 64>::THREADS, fa::FwdCfg<128, 64>::SMEM_BYTES, s>>>(mq, mk64, mv64, o, LSE, BH, N, sl2, rescale, fa::FwdNoList{0});
    }
    return launch_status();
  }
  if (d == 64) {
    if (causal) fa::fa_fwd_kernel<64, true><<<grid, fa::FwdCfg<64>::THREADS, fa::FwdCfg<64>::SMEM_BYTES, s>>>(mq, mk, mv, o, LSE, BH, N, sl2, rescale, ul);
    else fa::fa_fwd_kernel<64, false><<<grid, fa::FwdCfg<64>::THREADS, fa::FwdCfg<64>::SMEM_BYTES, s>>>(mq, mk, mv, o, LSE, BH, N, sl2, rescale, fa::FwdNoList{0});
  } else {
    if (causal) fa::fa_fwd_kernel<128, true><<<grid, fa::FwdCfg<128>::THREADS, fa::FwdCfg<128>::SMEM_BYTES, s>>>(mq, mk, mv, o, LSE, BH, N, sl2, rescale, ul);
    else fa::fa_fwd_kernel<128, false><<<grid, fa::FwdCfg<128>::THREADS, fa::FwdCfg<128>::SMEM_BYTES, s>>>(mq, mk, mv, o, LSE, BH, N, sl2, rescale, fa::FwdNoList{0});
  }
  return launch_status();
}

// ---------------------------------------------------------------------------
// standard (unfused) forward: S and P through HBM
// ---------------------------------------------------------------------------
static size_t unfused_rows_padded(int N) { return (static_cast<size_t>(N) + 127) / 128 * 128; }

size_t fa_fwd_unfused_workspace_bytes(int B, int H, int N, int d) {
  if (check_sizes(B, H, N, d)) return 0;
  const size_t nr = unfused_rows_padded(N);
  return static_cast<size_t>(B) * H * nr * nr * 2;
}

int fa_fwd_unfused(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int N, int d,
                   int causal, float scale, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_sizes(B, H, N, d);
  if (rc) return rc;
  if (!Q || !K || !V || !O || !LSE) return FA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE)) return FA_ERR_ALIGNMENT;
  bool scale_ok = false;
  const float sc = effective_scale(scale, d, &scale_ok);
  if (!scale_ok) return FA_ERR_INVALID_ARG;
  const size_t need = fa_fwd_unfused_workspace_bytes(B, H, N, d);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return FA_ERR_WORKSPACE;
  const int BH = B * H;
  const long long nt = static_cast<long long>(unfused_rows_padded(N) / 128);
  if (static_cast<long long>(BH) * nt * nt > 0x7fffffffLL) return FA_ERR_INVALID_ARG;  // grid limit
  const size_t tbytes = static_cast<size_t>(BH) * N * d * 2, lbytes = static_cast<size_t>(BH) * N * 4;
  const Range rq{(uintptr_t)Q, (uintptr_t)Q + tbytes}, rk{(uintptr_t)K, (uintptr_t)K + tbytes},
      rv{(uintptr_t)V, (uintptr_t)V + tbytes}, ro{(uintptr_t)O, (uintptr_t)O + tbytes},
      rl{(uintptr_t)LSE, (uintptr_t)LSE + lbytes}, rw{(uintptr_t)workspace, (uintptr_t)workspace + need};
  const Range ins[3] = {rq, rk, rv};
  for (int b = 0; b < 3; ++b)
    if (overlaps(ro, ins[b]) || overlaps(rl, ins[b])) return FA_ERR_INVALID_ARG;
  if (overlaps(ro, rl)) return FA_ERR_INVALID_ARG;
  if (overlaps(rw, rq) || overlaps(rw, rk) || overlaps(rw, rv) || overlaps(rw, ro) || overlaps(rw, rl))
    return FA_ERR_WORKSPACE;
  int sms = 0;
  if ((rc = device_ready(&sms))) return rc;
  if (!is_device_ptr(Q, tbytes) || !is_device_ptr(K, tbytes) || !is_device_ptr(V, tbytes) ||
      !is_device_ptr(O, tbytes) || !is_device_ptr(LSE, lbytes) || !is_device_ptr(workspace, need))
    return FA_ERR_UNSUPPORTED_DEVICE;
  const int Nr = static_cast<int>(nt * 128);
  CUtensorMap mq, mk, mp, mv;
  if (!make_map(&mq, Q, BH, N, d, 128) || !make_map(&mk, K, BH, N, d, 128) ||
      !make_map(&mp, workspace, BH, Nr, Nr, 128) || !make_map(&mv, V, BH, N, d, 64))
    return encode_failed();
  clear_stale_error();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* S = static_cast<__half*>(workspace);
  auto* o = static_cast<__nv_bfloat16*>(O);
  const unsigned grid_s = static_cast<unsigned>(BH * nt * nt), grid_pv = static_cast<unsigned>(BH * nt);
  const long long rows = static_cast<long long>(BH) * N;
  const unsigned grid_sm = static_cast<unsigned>((rows + fa::kUnfSoftmaxRows - 1) / fa::kUnfSoftmaxRows);
  if (d == 64) {
    fa::fa_unf_scores_kernel<64><<<grid_s, 128, fa::UnfScoresCfg<64>::SMEM_BYTES, s>>>(mq, mk, S, static_cast<int>(nt), Nr, sc);
    fa::fa_unf_softmax_kernel<<<grid_sm, 256, 0, s>>>(S, LSE, rows, N, Nr, causal ? 1 : 0);
    fa::fa_unf_pv_kernel<64><<<grid_pv, 128, fa::UnfPvCfg<64>::SMEM_BYTES, s>>>(mp, mv, o, N, Nr);
  } else {
    fa::fa_unf_scores_kernel<128><<<grid_s, 128, fa::UnfScoresCfg<128>::SMEM_BYTES, s>>>(mq, mk, S, static_cast<int>(nt), Nr, sc);
    fa::fa_unf_softmax_kernel<<<grid_sm, 256, 0, s>>>(S, LSE, rows, N, Nr, causal ? 1 : 0);
    fa::fa_unf_pv_kernel<128><<<grid_pv, 128, fa::UnfPvCfg<128>::SMEM_BYTES, s>>>(mp, mv, o, N, Nr);
  }
  return launch_status();
}

const char* fa_bwd_dkdv_kernel_name(int d) {
  if (d != 64 && d != 128) return nullptr;
  return "fa_bwd_fused_kernel";
}

// Workspace of the backward: D (fp32 [B*H*N], padded to 256 bytes), then the
// fp32 dQ accumulator [B*H*N*d] of the fused form.
static size_t bwd_d_bytes(int B, int H, int N) {
  const size_t dbytes = static_cast<size_t>(B) * H * N * 4;
  return (dbytes + 255) & ~static_cast<size_t>(255);
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (check_sizes(B, H, N, d)) return 0;
  return bwd_d_bytes(B, H, N) + static_cast<size_t>(B) * H * N * d * 4;
}

// The backward in either form.  fused: one kernel computes dK, dV and the dQ
// partials (fp32 accumulator in the workspace), then a convert pass; else the
// deterministic form: dK/dV kernel and a dQ kernel that recomputes S and dP.
// `need` is the workspace the form uses (validated against workspace_bytes).
static int bwd_launch(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                      void* dQ, void* dK, void* dV, int B, int H, int N, int d, int causal, float scale,
                      void* workspace, size_t workspace_bytes, void* stream, bool fused) {
  int rc = check_sizes(B, H, N, d);
  if (rc) return rc;
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV) return FA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) || !aligned16(LSE) ||
      !aligned16(dQ) || !aligned16(dK) || !aligned16(dV))
    return FA_ERR_ALIGNMENT;
  const size_t need = fused ? fa_bwd_workspace_bytes(B, H, N, d) : bwd_d_bytes(B, H, N);
  if (!workspace || !aligned16(workspace) || workspace_bytes < need) return FA_ERR_WORKSPACE;
  bool scale_ok = false;
  const float sc = effective_scale(scale, d, &scale_ok);
  if (!scale_ok) return FA_ERR_INVALID_ARG;
  const size_t tbytes = static_cast<size_t>(B) * H * N * d * 2, lbytes = static_cast<size_t>(B) * H * N * 4;
  const Range ins[6] = {{(uintptr_t)Q, (uintptr_t)Q + tbytes},   {(uintptr_t)K, (uintptr_t)K + tbytes},
                        {(uintptr_t)V, (uintptr_t)V + tbytes},   {(uintptr_t)O, (uintptr_t)O + tbytes},
                        {(uintptr_t)dO, (uintptr_t)dO + tbytes}, {(uintptr_t)LSE, (uintptr_t)LSE + lbytes}};
  const Range outs[4] = {{(uintptr_t)dQ, (uintptr_t)dQ + tbytes},
                         {(uintptr_t)dK, (uintptr_t)dK + tbytes},
                         {(uintptr_t)dV, (uintptr_t)dV + tbytes},
                         {(uintptr_t)workspace, (uintptr_t)workspace + need}};
  for (int a = 0; a < 4; ++a) {
    for (int b = 0; b < 6; ++b)
      if (overlaps(outs[a], ins[b])) return a == 3 ? FA_ERR_WORKSPACE : FA_ERR_INVALID_ARG;
    for (int b = a + 1; b < 4; ++b)
      if (overlaps(outs[a], outs[b])) return b == 3 ? FA_ERR_WORKSPACE : FA_ERR_INVALID_ARG;
  }
  int sms = 0;
  if ((rc = device_ready(&sms))) return rc;
  const void* ptrs[10] = {Q, K, V, O, dO, LSE, dQ, dK, dV, workspace};
  const size_t sizes[10] = {tbytes, tbytes, tbytes, tbytes, tbytes, lbytes, tbytes, tbytes, tbytes, need};
  for (int i = 0; i < 10; ++i)
    if (!is_device_ptr(ptrs[i], sizes[i])) return FA_ERR_UNSUPPORTED_DEVICE;
  const int BH = B * H;
  CUtensorMap mq64, mdo64, mk128, mv128, mq128, mdo128, mk64, mv64;
  if (!make_map(&mq64, Q, BH, N, d, 64) || !make_map(&mdo64, dO, BH, N, d, 64) ||
      !make_map(&mk128, K, BH, N, d, 128) || !make_map(&mv128, V, BH, N, d, 128))
    return encode_failed();
  if (!fused && (!make_map(&mq128, Q, BH, N, d, 128) || !make_map(&mdo128, dO, BH, N, d, 128) ||
                 !make_map(&mk64, K, BH, N, d, 64) || !make_map(&mv64, V, BH, N, d, 64)))
    return encode_failed();
  // the fused kernel's query tiles: boxes of its BQ rows
  CUtensorMap mqf, mdof;
  const int fused_bq = d == 64 ? fa::FusedCfg<64>::BQ : fa::FusedCfg<128>::BQ;
  if (fused && (!make_map(&mqf, Q, BH, N, d, fused_bq) || !make_map(&mdof, dO, BH, N, d, fused_bq)))
    return encode_failed();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  clear_stale_error();
  float* Dvec = static_cast<float*>(workspace);
  float* dqacc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + bwd_d_bytes(B, H, N));
  const long long rows = static_cast<long long>(BH) * N;
  const float sl2 = sc * fa::kLog2e;
  auto* dq = static_cast<__nv_bfloat16*>(dQ);
  auto* dk = static_cast<__nv_bfloat16*>(dK);
  auto* dv = static_cast<__nv_bfloat16*>(dV);
  auto* o = static_cast<const __nv_bfloat16*>(O);
  auto* dob = static_cast<const __nv_bfloat16*>(dO);
  cudaEvent_t ev[4];
  {
    std::lock_guard<std::mutex> lock(g_events_mu);
    for (int e = 0; e < 4; ++e) ev[e] = g_phase_events[e];
  }
  auto mark = [&](int e) {
    if (ev[e]) cudaEventRecord(ev[e], s);
  };
  const int grid_kv = BH * ((N + 127) / 128);
  const int grid_q = BH * ((N + 127) / 128);
  // the fused kernel is persistent: one CTA per SM, each walking its units
  const int grid_fused = grid_kv < sms ? grid_kv : sms;
  fa::UnitList bul;  // with the mask: this shape's unit lists (n = 0: serpentine deal)
  bul.n = 0;
  if (fused && causal) causal_bwd_unit_list(&bul, BH, N, d, grid_fused);
  const unsigned grid_pre = static_cast<unsigned>((rows * (d / 8) + 255) / 256);
  const unsigned grid_cvt = static_cast<unsigned>((rows * d / 8 + 255) / 256);
  mark(0);
  if (d == 64) {
    if (fused) {
      fa::fa_bwd_preprocess_kernel<64, true><<<grid_pre, 256, 0, s>>>(o, dob, Dvec, rows, dqacc);
      mark(1);
      if (causal) fa::fa_bwd_fused_kernel<64, true><<<grid_fused, fa::FusedCfg<64>::THREADS, fa::FusedCfg<64>::SMEM_BYTES, s>>>(mqf, mk128, mv128, mdof, LSE, Dvec, dk, dv, dqacc, BH, N, sc, sl2, bul);
      else fa::fa_bwd_fused_kernel<64, false><<<grid_fused, fa::FusedCfg<64>::THREADS, fa::FusedCfg<64>::SMEM_BYTES, s>>>(mqf, mk128, mv128, mdof, LSE, Dvec, dk, dv, dqacc, BH, N, sc, sl2, fa::NoUnitList{0});
      mark(2);
      fa::fa_bwd_dq_convert_kernel<<<grid_cvt, 256, 0, s>>>(dqacc, dq, rows * d / 8, sc);
    } else {
      fa::fa_bwd_preprocess_kernel<64><<<grid_pre, 256, 0, s>>>(o, dob, Dvec, rows);
      mark(1);
      if (causal) fa::fa_bwd_dkdv_kernel<64, true><<<grid_kv, fa::DkdvCfg<64>::THREADS, fa::DkdvCfg<64>::SMEM_BYTES, s>>>(mq64, mk128, mv128, mdo64, LSE, Dvec, dk, dv, N, sc, sl2);
      else fa::fa_bwd_dkdv_kernel<64, false><<<grid_kv, fa::DkdvCfg<64>::THREADS, fa::DkdvCfg<64>::SMEM_BYTES, s>>>(mq64, mk128, mv128, mdo64, LSE, Dvec, dk, dv, N, sc, sl2);
      mark(2);
      if (causal) fa::fa_bwd_dq_kernel<64, true><<<grid_q, fa::DqCfg<64>::THREADS, fa::DqCfg<64>::SMEM_BYTES, s>>>(mq128, mk64, mv64, mdo128, LSE, Dvec, dq, N, sc, sl2);
      else fa::fa_bwd_dq_kernel<64, false><<<grid_q, fa::DqCfg<64>::THREADS, fa::DqCfg<64>::SMEM_BYTES, s>>>(mq128, mk64, mv64, mdo128, LSE, Dvec, dq, N, sc, sl2);
    }
  } else {
    if (fused) {
      fa::fa_bwd_preprocess_kernel<128, true><<<grid_pre, 256, 0, s>>>(o, dob, Dvec, rows, dqacc);
      mark(1);
      if (causal) fa::fa_bwd_fused_kernel<128, true><<<grid_fused, fa::FusedCfg<128>::THREADS, fa::FusedCfg<128>::SMEM_BYTES, s>>>(mqf, mk128, mv128, mdof, LSE, Dvec, dk, dv, dqacc, BH, N, sc, sl2, bul);
      else fa::fa_bwd_fused_kernel<128, false><<<grid_fused, fa::FusedCfg<128>::THREADS, fa::FusedCfg<128>::SMEM_BYTES, s>>>(mqf, mk128, mv128, mdof, LSE, Dvec, dk, dv, dqacc, BH, N, sc, sl2, fa::NoUnitList{0});
      mark(2);
      fa::fa_bwd_dq_convert_kernel<<<grid_cvt, 256, 0, s>>>(dqacc, dq, rows * d / 8, sc);
    } else {
      fa::fa_bwd_preprocess_kernel<128><<<grid_pre, 256, 0, s>>>(o, dob, Dvec, rows);
      mark(1);
      if (causal) fa::fa_bwd_dkdv_kernel<128, true><<<grid_kv, fa::DkdvCfg<128>::THREADS, fa::DkdvCfg<128>::SMEM_BYTES, s>>>(mq64, mk128, mv128, mdo64, LSE, Dvec, dk, dv, N, sc, sl2);
      else fa::fa_bwd_dkdv_kernel<128, false><<<grid_kv, fa::DkdvCfg<128>::THREADS, fa::DkdvCfg<128>::SMEM_BYTES, s>>>(mq64, mk128, mv128, mdo64, LSE, Dvec, dk, dv, N, sc, sl2);
      mark(2);
      if (causal) fa::fa_bwd_dq_kernel<128, true><<<grid_q, fa::DqCfg<128>::THREADS, fa::DqCfg<128>::SMEM_BYTES, s>>>(mq128, mk64, mv64, mdo128, LSE, Dvec, dq, N, sc, sl2);
      else fa::fa_bwd_dq_kernel<128, false><<<grid_q, fa::DqCfg<128>::THREADS, fa::DqCfg<128>::SMEM_BYTES, s>>>(mq128, mk64, mv64, mdo128, LSE, Dvec, dq, N, sc, sl2);
    }
  }
  mark(3);
  return launch_status();
}

int fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE, void* dQ,
           void* dK, void* dV, int B, int H, int N, int d, int causal, float scale, void* workspace,
           size_t workspace_bytes, void* stream) {
  return bwd_launch(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, causal, scale, workspace, workspace_bytes, stream,
                    true);
}

int fa_bwd_deterministic(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                         const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int N, int d, int causal,
                         float scale, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_launch(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, causal, scale, workspace, workspace_bytes, stream,
                    false);
}

static unsigned int g_last_error_word = 0;

void fa_bwd_set_phase_events(void* e0, void* e1, void* e2, void* e3) {
  std::lock_guard<std::mutex> lock(g_events_mu);
  g_phase_events[0] = static_cast<cudaEvent_t>(e0);
  g_phase_events[1] = static_cast<cudaEvent_t>(e1);
  g_phase_events[2] = static_cast<cudaEvent_t>(e2);
  g_phase_events[3] = static_cast<cudaEvent_t>(e3);
}

int fa_sync_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    g_last_cuda_error = static_cast<int>(e);
    return FA_ERR_LAUNCH;
  }
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, fa::g_error_word, sizeof(word)) != cudaSuccess) return FA_ERR_LAUNCH;
  if (word != 0) {
    const unsigned int zero = 0;
    g_last_error_word = word;
    if (cudaMemcpyToSymbol(fa::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_LAUNCH;
    return FA_ERR_TIMEOUT;
  }
  return FA_OK;
}

unsigned int fa_last_error_word(void) { return g_last_error_word; }

int fa_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"

namespace fa {
// One warp initialises a barrier that nothing arrives on and waits for it
// with a short wall-clock limit; the wait records the timeout and returns.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_wait_slow(b, 0, 255u, limit_ns);
}
}  // namespace fa

extern "C" int fa_selftest_wait_timeout(unsigned int limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 10000000u) return FA_ERR_INVALID_ARG;
  int sms = 0;
  int rc = device_ready(&sms);
  if (rc) return rc;
  clear_stale_error();
  fa::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_us) * 1000ull);
  return launch_status();
}

// ---------------------------------------------------------------------------
// fa_bwd_noalloc: the backward with its D vector in a fixed device array, for
// callers that cannot allocate device memory.
// ---------------------------------------------------------------------------
namespace {
// FA_NOALLOC_MAX_ROWS fp32 entries; every device that loads the library holds
// it until the process exits.  In host code this name is only a stand-in:
// kernels get the device address from cudaGetSymbolAddress below.
__device__ __align__(256) float g_noalloc_d[FA_NOALLOC_MAX_ROWS];
void* g_noalloc_addr[kMaxDevices] = {};
void* g_noalloc_ctx[kMaxDevices] = {};  // the CUDA context each address belongs to
std::mutex g_noalloc_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
// The current thread's CUDA context (the device's primary context once the
// runtime has bound it), or null.
void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!fn || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}
}  // namespace

extern "C" int fa_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                              const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int N, int d,
                              int causal, float scale, void* stream) {
  int rc = check_sizes(B, H, N, d);
  if (rc) return rc;
  if (static_cast<long long>(B) * H * N > FA_NOALLOC_MAX_ROWS) return FA_ERR_TOO_LARGE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA_ERR_UNSUPPORTED_DEVICE;
  }
  // Binds the device's primary context to this thread if it has none yet, so
  // that the context looked up below is the one the kernels will run in.
  if (cudaSetDevice(dev) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_UNSUPPORTED_DEVICE;
  }
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    void* ctx = current_context();
    // set-up, once per device (and again after a device reset gave it a new
    // context), with that device current
    if (!g_noalloc_addr[dev] || ctx != g_noalloc_ctx[dev]) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_d);
      if (e != cudaSuccess || !p) {
        g_last_cuda_error = static_cast<int>(e);
        cudaGetLastError();
        return FA_ERR_LAUNCH;
      }
      g_noalloc_addr[dev] = p;
      g_noalloc_ctx[dev] = ctx;
    }
    scratch = g_noalloc_addr[dev];
  }
  // The deterministic form needs only D, which its first kernel writes in full
  // before anything reads it, so the array needs no clearing between calls.
  return bwd_launch(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, causal, scale, scratch,
                    static_cast<size_t>(FA_NOALLOC_MAX_ROWS) * sizeof(float), stream, false);
}

// ---------------------------------------------------------------------------
// fa_fwd_bwd_host: forward + backward from host memory to host memory, the
// PCIe copies overlapped with the kernels
// ---------------------------------------------------------------------------
namespace {
constexpr int kHostSlots = 3;  // copy-in of group c, kernels of c-1 and copy-out of c-2 run at once

// The library's own streams and events for the pipeline, one set per device,
// created at the first call on that device and kept until the process exits.
struct HostPipe {
  bool ready = false;
  cudaStream_t s_in = nullptr, s_run = nullptr, s_out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t ev_in[kHostSlots] = {}, ev_run[kHostSlots] = {}, ev_out[kHostSlots] = {};
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_pipe_mu;  // held for a whole call's enqueue: the streams and events are shared

bool host_pipe_ready(HostPipe& p) {
  if (p.ready) return true;
  bool ok = cudaStreamCreateWithFlags(&p.s_in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p.s_run, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p.s_out, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.done, cudaEventDisableTiming) == cudaSuccess;
  for (int i = 0; i < kHostSlots && ok; ++i)
    ok = cudaEventCreateWithFlags(&p.ev_in[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p.ev_run[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p.ev_out[i], cudaEventDisableTiming) == cudaSuccess;
  p.ready = ok;
  return ok;
}

// One slot of the device workspace: one head group's inputs, outputs and
// backward workspace, each region 256-byte aligned.
struct HostSlot {
  size_t q, k, v, dO, o, lse, dq, dk, dv, ws, ws_bytes, total;
};
HostSlot host_slot(int hc, int N, int d) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t t = up(static_cast<size_t>(hc) * N * d * 2), l = up(static_cast<size_t>(hc) * N * 4);
  HostSlot s;
  size_t off = 0;
  s.q = off, off += t;
  s.k = off, off += t;
  s.v = off, off += t;
  s.dO = off, off += t;
  s.o = off, off += t;
  s.lse = off, off += l;
  s.dq = off, off += t;
  s.dk = off, off += t;
  s.dv = off, off += t;
  s.ws = off;
  s.ws_bytes = up(fa_bwd_workspace_bytes(1, hc, N, d));
  off += s.ws_bytes;
  s.total = off;
  return s;
}

int heads_per_group(int BH, int groups) {
  const int g = groups < BH ? groups : BH;
  return (BH + g - 1) / g;
}
}  // namespace

extern "C" int fa_unit_lists(int kind, int B, int H, int N, int d, int grid, unsigned short* start,
                             unsigned short* order, int max_units) {
  if ((kind != 0 && kind != 1) || check_sizes(B, H, N, d) || grid < 1 || grid > fa::UnitList::kMaxCtas || !start ||
      !order)
    return FA_ERR_INVALID_ARG;
  const int BH = B * H;
  fa::UnitList L;
  L.n = 0;
  const bool built = kind == 0 ? build_unit_list(&L, BH, N, d, 128, grid) : build_bwd_unit_list(&L, BH, N, d, grid);
  if (!built) return 0;
  if (max_units < L.n) return FA_ERR_INVALID_ARG;
  for (int c = 0; c <= grid; ++c) start[c] = L.start[c];
  for (int i = 0; i < L.n; ++i) order[i] = L.order[i];
  return L.n;
}

extern "C" size_t fa_fwd_bwd_host_workspace_bytes(int B, int H, int N, int d, int groups) {
  if (check_sizes(B, H, N, d) || groups < 1) return 0;
  return kHostSlots * host_slot(heads_per_group(B * H, groups), N, d).total;
}

extern "C" int fa_fwd_bwd_host(const void* Q, const void* K, const void* V, const void* dO, void* O, float* LSE,
                               void* dQ, void* dK, void* dV, int B, int H, int N, int d, int causal, float scale,
                               int groups, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_sizes(B, H, N, d);
  if (rc) return rc;
  if (groups < 1) return FA_ERR_INVALID_ARG;
  if (!Q || !K || !V || !dO || !O || !LSE || !dQ || !dK || !dV) return FA_ERR_INVALID_ARG;
  bool scale_ok = false;
  (void)effective_scale(scale, d, &scale_ok);
  if (!scale_ok) return FA_ERR_INVALID_ARG;
  const size_t need = fa_fwd_bwd_host_workspace_bytes(B, H, N, d, groups);
  if (!workspace || !aligned16(workspace) || workspace_bytes < need) return FA_ERR_WORKSPACE;
  const size_t tbytes = static_cast<size_t>(B) * H * N * d * 2, lbytes = static_cast<size_t>(B) * H * N * 4;
  const Range ins[4] = {{(uintptr_t)Q, (uintptr_t)Q + tbytes},
                        {(uintptr_t)K, (uintptr_t)K + tbytes},
                        {(uintptr_t)V, (uintptr_t)V + tbytes},
                        {(uintptr_t)dO, (uintptr_t)dO + tbytes}};
  const Range outs[5] = {{(uintptr_t)O, (uintptr_t)O + tbytes},
                         {(uintptr_t)LSE, (uintptr_t)LSE + lbytes},
                         {(uintptr_t)dQ, (uintptr_t)dQ + tbytes},
                         {(uintptr_t)dK, (uintptr_t)dK + tbytes},
                         {(uintptr_t)dV, (uintptr_t)dV + tbytes}};
  for (int a = 0; a < 5; ++a) {
    for (int b = 0; b < 4; ++b)
      if (overlaps(outs[a], ins[b])) return FA_ERR_INVALID_ARG;
    for (int b = a + 1; b < 5; ++b)
      if (overlaps(outs[a], outs[b])) return FA_ERR_INVALID_ARG;
  }
  int sms = 0;
  if ((rc = device_ready(&sms))) return rc;
  if (!is_device_ptr(workspace, need)) return FA_ERR_UNSUPPORTED_DEVICE;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe& p = g_pipe[dev];
  if (!host_pipe_ready(p)) {
    g_last_cuda_error = static_cast<int>(cudaGetLastError());
    return FA_ERR_LAUNCH;
  }
  clear_stale_error();
  const int BH = B * H, hc = heads_per_group(BH, groups);
  const int ng = (BH + hc - 1) / hc;
  const HostSlot L = host_slot(hc, N, d);
  const size_t head_t = static_cast<size_t>(N) * d * 2, head_l = static_cast<size_t>(N) * 4;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the pipeline starts after the work already queued on the caller's stream
  cudaEventRecord(p.start, s);
  cudaStreamWaitEvent(p.s_in, p.start, 0);
  cudaStreamWaitEvent(p.s_run, p.start, 0);
  cudaStreamWaitEvent(p.s_out, p.start, 0);
  auto dptr = [&](int slot, size_t off) { return static_cast<uint8_t*>(workspace) + slot * L.total + off; };
  for (int c = 0; c < ng; ++c) {
    const int slot = c % kHostSlots;
    const int h0 = c * hc, hn = (BH - h0) < hc ? (BH - h0) : hc;
    const size_t nt = hn * head_t, nl = hn * head_l, ot = h0 * head_t, ol = h0 * head_l;
    // copies in: the slot is free once group c - kHostSlots has been copied out
    if (c >= kHostSlots) cudaStreamWaitEvent(p.s_in, p.ev_out[slot], 0);
    const void* srcs[4] = {Q, K, V, dO};
    const size_t dsts[4] = {L.q, L.k, L.v, L.dO};
    for (int i = 0; i < 4; ++i)
      cudaMemcpyAsync(dptr(slot, dsts[i]), static_cast<const uint8_t*>(srcs[i]) + ot, nt, cudaMemcpyDefault,
                      p.s_in);
    cudaEventRecord(p.ev_in[slot], p.s_in);
    // forward and backward of the group's heads (B = 1, H = hn: the heads are contiguous)
    cudaStreamWaitEvent(p.s_run, p.ev_in[slot], 0);
    rc = fa_fwd(dptr(slot, L.q), dptr(slot, L.k), dptr(slot, L.v), dptr(slot, L.o),
                reinterpret_cast<float*>(dptr(slot, L.lse)), 1, hn, N, d, causal, scale, p.s_run);
    if (!rc)
      rc = fa_bwd(dptr(slot, L.q), dptr(slot, L.k), dptr(slot, L.v), dptr(slot, L.o), dptr(slot, L.dO),
                  reinterpret_cast<const float*>(dptr(slot, L.lse)), dptr(slot, L.dq), dptr(slot, L.dk),
                  dptr(slot, L.dv), 1, hn, N, d, causal, scale, dptr(slot, L.ws), L.ws_bytes, p.s_run);
    if (rc) break;  // no copy out of this group; the work already queued is still joined below
    cudaEventRecord(p.ev_run[slot], p.s_run);
    // copies out
    cudaStreamWaitEvent(p.s_out, p.ev_run[slot], 0);
    cudaMemcpyAsync(static_cast<uint8_t*>(O) + ot, dptr(slot, L.o), nt, cudaMemcpyDefault, p.s_out);
    cudaMemcpyAsync(reinterpret_cast<uint8_t*>(LSE) + ol, dptr(slot, L.lse), nl, cudaMemcpyDefault, p.s_out);
    cudaMemcpyAsync(static_cast<uint8_t*>(dQ) + ot, dptr(slot, L.dq), nt, cudaMemcpyDefault, p.s_out);
    cudaMemcpyAsync(static_cast<uint8_t*>(dK) + ot, dptr(slot, L.dk), nt, cudaMemcpyDefault, p.s_out);
    cudaMemcpyAsync(static_cast<uint8_t*>(dV) + ot, dptr(slot, L.dv), nt, cudaMemcpyDefault, p.s_out);
    cudaEventRecord(p.ev_out[slot], p.s_out);
  }
  // the caller's stream continues once everything this call queued is done
  // (on error too, so that no copy into the caller's buffers outlives the
  // stream order the caller sees)
  cudaEventRecord(p.done, p.s_in);
  cudaStreamWaitEvent(p.s_out, p.done, 0);
  cudaEventRecord(p.done, p.s_run);
  cudaStreamWaitEvent(p.s_out, p.done, 0);
  cudaEventRecord(p.done, p.s_out);
  cudaStreamWaitEvent(s, p.done, 0);
  const int st = launch_status();
  return rc ? rc : st;
}
