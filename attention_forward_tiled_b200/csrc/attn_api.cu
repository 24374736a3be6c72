// attn_api.cu -- the C ABI of libattn.so (declared in include/attn.h).
//
// Host side only: argument validation, tensor-map encoding for the
// tensor-memory accelerator, launch configuration, the split-KV workspace and
// the device status word.  Every arithmetic step of the attention forward runs
// in the kernels of prefill_sm100.cuh and decode_sm100.cuh; there is no CPU
// fallback.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "backward_sm100.cuh"
#include "relpos_sm100.cuh"
#include "decode_mq_sm100.cuh"
#include "decode_sm100.cuh"
#include "indexer_sm100.cuh"
#include "prefill_sm100.cuh"

using namespace attn_b200;

// Device status word: kernels record ATTN_ERR_TIMEOUT / ATTN_ERR_RANGE here instead of trapping.
__device__ int g_attn_status = 0;

// Fixed scratch of attn_fwd_decode_noalloc: the split partials live here instead of in
// a per-call allocation.  Every GPU that loads this library holds these 4 MiB until the
// process exits.  All calls share it and it keeps the last call's contents.
constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

namespace {

constexpr int kVersion = 10000;  // 1.0.0
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded wait
constexpr int kMaxDevices = 64;
// Prefill scheduling group: units of 16 heads are handed out together (heaviest causal
// units first), so the K/V being read stay in L2 (16 heads x 4096 keys x d 128 x 2 x 2 B
// = 32 MB) while the group is long enough to even out the causal unit sizes over SMs.
// (12 or 24 heads per group measured slower or equal on the causal workloads.)
constexpr int kHeadsPerGroup = 16;

std::atomic<int> g_inject{0};
std::atomic<unsigned long long> g_timeout_ns{kDefaultTimeoutNs};

struct DeviceState {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
  int* status_ptr = nullptr;
  bool attr_set[32] = {};  // per kernel instantiation: max dynamic shared memory raised
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mutex;

// Device address of g_noalloc_scratch, looked up once per device (with it current).
float* g_noalloc_scratch_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mutex;

int noalloc_scratch_ptr(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return ATTN_ERR_CUDA;
    g_noalloc_scratch_ptr[dev] = static_cast<float*>(ptr);
  }
  *out = g_noalloc_scratch_ptr[dev];
  return ATTN_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Probe the current device once: sm_100 check, SM count, status-word address.
int device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceState& s = g_dev[dev];
  if (!s.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    s.supported = (major == 10 && minor == 0);
    s.sm_count = sms;
    if (s.supported) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_attn_status) != cudaSuccess) return ATTN_ERR_CUDA;
      s.status_ptr = static_cast<int*>(ptr);
    }
    s.probed = true;
  }
  if (!s.supported) return ATTN_ERR_UNSUPPORTED;
  *out = &s;
  return ATTN_OK;
}

// Raise the dynamic shared-memory limit of a kernel once per device.
template <typename Kernel>
int ensure_smem_attr(DeviceState* ds, int slot, Kernel kernel, int bytes) {
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (ds->attr_set[slot]) return ATTN_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return ATTN_ERR_CUDA;
  ds->attr_set[slot] = true;
  return ATTN_OK;
}

// 4-D view (d, H, N, B) of a contiguous [B, N, H, d] tensor; box (64, 1, box_rows, 1), 128B swizzle.
int encode_bnhd(CUtensorMap* map, const void* ptr, int B, int N, int H, int d, int dtype,
                int box_rows = 128) {
  EncodeTiledFn encode = get_encode_fn();
  if (!encode) return ATTN_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2,
                                 (cuuint64_t)N * H * d * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType ty =
      dtype == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = encode(map, ty, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// 3-D view (d, rows, B) of a contiguous [B, rows, d] tensor; box (64, 128, 1), 128B swizzle.
int encode_rows3d(CUtensorMap* map, const void* ptr, int B, long long rows, int d, int dtype,
                  int box_rows = 128) {
  EncodeTiledFn encode = get_encode_fn();
  if (!encode) return ATTN_ERR_CUDA;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType ty =
      dtype == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = encode(map, ty, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// 4-D view (d, H, N, B) of a contiguous fp32 [B, N, H, d] tensor; box (d, 1, box_rows, 1),
// no swizzle (the backward's dQ accumulator, written by TMA reduce-adds).
int encode_f32_bnhd(CUtensorMap* map, void* ptr, int B, int N, int H, int d, int box_rows) {
  EncodeTiledFn encode = get_encode_fn();
  if (!encode) return ATTN_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 4, (cuuint64_t)H * d * 4, (cuuint64_t)N * H * d * 4};
  const cuuint32_t box[4] = {(cuuint32_t)d, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ptr, dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// 3-D view (P, T, B) of a contiguous f16 [B, T, P] pool mask; box (256 keys, tokens, 1), no
// swizzle.  Needs P a multiple of 8 (16-byte row pitch) and a 16-byte aligned base.
int encode_mask3d(CUtensorMap* map, const void* ptr, int B, int T, int P, int box_tokens) {
  EncodeTiledFn encode = get_encode_fn();
  if (!encode) return ATTN_ERR_CUDA;
  const cuuint64_t dims[3] = {(cuuint64_t)P, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)P * 2, (cuuint64_t)T * P * 2};
  const cuuint32_t box[3] = {256, (cuuint32_t)box_tokens, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
                      estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Shared argument checks of every entry point (nothing is enqueued on failure).
int validate(const void* q, const void* k, const void* v, const void* out, const float* lse,
             int B, int H, int Nq, int Nk, int d, int causal, float scale, int dtype) {
  if (!q || !k || !v || !out) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (dtype != ATTN_F16 && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  auto misaligned = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) != 0; };
  if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(out, 16))
    return ATTN_ERR_INVALID_ARG;
  if (lse && misaligned(lse, 4)) return ATTN_ERR_INVALID_ARG;
  // tensor-map limits: the batch stride (N*H*d*2 bytes) must stay below 2^40
  const unsigned long long row_bytes = (unsigned long long)H * d * 2;
  if ((unsigned long long)Nq * row_bytes >= (1ull << 40) ||
      (unsigned long long)Nk * row_bytes >= (1ull << 40))
    return ATTN_ERR_INVALID_ARG;
  const size_t q_bytes = (size_t)B * Nq * row_bytes;
  const size_t kv_bytes = (size_t)B * Nk * row_bytes;
  const size_t lse_bytes = (size_t)B * H * Nq * sizeof(float);
  if (overlaps(out, q_bytes, q, q_bytes) || overlaps(out, q_bytes, k, kv_bytes) ||
      overlaps(out, q_bytes, v, kv_bytes))
    return ATTN_ERR_INVALID_ARG;
  if (lse && (overlaps(lse, lse_bytes, out, q_bytes) || overlaps(lse, lse_bytes, q, q_bytes) ||
              overlaps(lse, lse_bytes, k, kv_bytes) || overlaps(lse, lse_bytes, v, kv_bytes)))
    return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

template <int D, bool BF16>
int launch_prefill(DeviceState* ds, const void* q, const void* k, const void* v, void* out,
                   float* lse, int B, int H, int Nq, int Nk, int causal, float scale,
                   cudaStream_t stream) {
  using C = PrefillCfg<D>;
  auto kernel = attn_prefill_kernel<D, BF16>;
  const int slot = (D == 128 ? 0 : 1) + (BF16 ? 2 : 0);
  if (int rc = ensure_smem_attr(ds, slot, kernel, C::kSmemBytes)) return rc;
  PrefillParams p;
  const int dtype = BF16 ? ATTN_BF16 : ATTN_F16;
  if (int rc = encode_bnhd(&p.tm_q, q, B, Nq, H, D, dtype)) return rc;
  if (int rc = encode_bnhd(&p.tm_k, k, B, Nk, H, D, dtype)) return rc;
  if (int rc = encode_bnhd(&p.tm_v, v, B, Nk, H, D, dtype)) return rc;
  if (int rc = encode_bnhd(&p.tm_o, out, B, Nq, H, D, dtype)) return rc;
  p.out = out;
  p.lse = lse;
  p.status = ds->status_ptr;
  p.B = B;
  p.H = H;
  p.Nq = Nq;
  p.Nk = Nk;
  p.causal = causal;
  p.n_qpairs = (Nq + 255) / 256;
  p.group_heads = kHeadsPerGroup;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.inject = g_inject.load();
  p.timeout_ns = g_timeout_ns.load();
  const long long pairs = (long long)B * H * p.n_qpairs;
  // Equal-sized (non-causal) units end in a partial wave; when it would fill at most half
  // of the SMs, its pairs run as single-tile units, two per pair, in about half the time.
  const long long rem = pairs % ds->sm_count;
  p.n_split = (!causal && pairs > ds->sm_count && 2 * rem <= ds->sm_count) ? (int)rem : 0;
  const long long units = pairs + p.n_split;
  if (units >= (1LL << 31)) return ATTN_ERR_INVALID_ARG;
  kernel<<<dim3((unsigned)units), dim3(C::kThreads), C::kSmemBytes, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Split count for the decode kernel: minimise the largest per-CTA tile count
// (items are dealt round-robin to one persistent CTA per SM), preferring fewer splits;
// at most max_splits.
int choose_splits(long long BH, int ntiles, int grid, long long max_splits = 1LL << 30) {
  int best = 1;
  long long best_load = -1;
  for (int s = 1; s <= ntiles && s <= max_splits; ++s) {
    const int tps = (ntiles + s - 1) / s;
    const int s_eff = (ntiles + tps - 1) / tps;
    if (s_eff != s) continue;
    const long long items = BH * s;
    const long long g = std::min<long long>(items, grid);
    const long long load = ((items + g - 1) / g) * tps;
    if (best_load < 0 || load * 100 < best_load * 98) {  // need a 2% gain to add splits
      best = s;
      best_load = load;
    }
  }
  return best;
}

template <int D, bool BF16>
int launch_decode(DeviceState* ds, const void* q, const void* k, const void* v, void* out,
                  float* lse, int B, int H, int Nk, float scale, int splits_req,
                  cudaStream_t stream) {
  using C = DecodeCfg<D>;
  auto kernel = attn_decode_partial_kernel<D, BF16>;
  const int slot = 4 + (D == 128 ? 0 : 1) + (BF16 ? 2 : 0);
  if (int rc = ensure_smem_attr(ds, slot, kernel, C::kSmemBytes)) return rc;
  const int ntiles = (Nk + 127) / 128;
  const long long BH = (long long)B * H;
  int splits = splits_req > 0 ? splits_req : choose_splits(BH, ntiles, ds->sm_count);
  if (splits < 1 || splits > ntiles) return ATTN_ERR_INVALID_ARG;
  const int tps = (ntiles + splits - 1) / splits;
  splits = (ntiles + tps - 1) / tps;  // no empty split
  const long long items = BH * splits;
  if (items >= (1LL << 31)) return ATTN_ERR_INVALID_ARG;

  DecodeParams p;
  const int dtype = BF16 ? ATTN_BF16 : ATTN_F16;
  if (int rc = encode_bnhd(&p.tm_k, k, B, Nk, H, D, dtype)) return rc;
  if (int rc = encode_bnhd(&p.tm_v, v, B, Nk, H, D, dtype)) return rc;
  float* part = nullptr;
  const size_t ws_bytes = (size_t)items * (D + 2) * sizeof(float);
  if (cudaMallocAsync(reinterpret_cast<void**>(&part), ws_bytes, stream) != cudaSuccess)
    return ATTN_ERR_CUDA;
  p.q = q;
  p.part = part;
  p.status = ds->status_ptr;
  p.B = B;
  p.H = H;
  p.Nk = Nk;
  p.splits = splits;
  p.tiles_per_split = tps;
  p.n_items = (int)items;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns.load();
  const int grid = (int)std::min<long long>(items, ds->sm_count);
  kernel<<<dim3(grid), dim3(C::kThreads), C::kSmemBytes, stream>>>(p);
  int rc = cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  if (rc == ATTN_OK) {
    attn_decode_combine_kernel<D, BF16>
        <<<dim3((unsigned)((BH + 3) / 4)), dim3(128), 0, stream>>>(part, out, lse, (int)BH, splits);
    rc = cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  if (cudaFreeAsync(part, stream) != cudaSuccess) rc = ATTN_ERR_CUDA;
  return rc;
}

// Paged cache: the same two kernels, the partial one reading each request's keys and
// values page by page through its block table (up to seq_lens[b] keys).
template <int D, bool BF16>
int launch_decode_paged(DeviceState* ds, const void* q, const void* k_cache, const void* v_cache,
                        const int* block_table, const int* seq_lens, void* out, float* lse, int B,
                        int H, int num_blocks, int page_size, int max_blocks, float scale,
                        int splits_req, cudaStream_t stream) {
  using C = DecodeCfg<D>;
  auto kernel = attn_decode_partial_kernel<D, BF16, true>;
  const int slot = 8 + (D == 128 ? 0 : 1) + (BF16 ? 2 : 0);
  if (int rc = ensure_smem_attr(ds, slot, kernel, C::kSmemBytes)) return rc;
  const int Nk = max_blocks * page_size;  // validated < 2^31
  const int ntiles = (Nk + 127) / 128;
  const long long BH = (long long)B * H;
  int splits = splits_req > 0 ? splits_req : choose_splits(BH, ntiles, ds->sm_count);
  if (splits < 1 || splits > ntiles) return ATTN_ERR_INVALID_ARG;
  const int tps = (ntiles + splits - 1) / splits;
  splits = (ntiles + tps - 1) / tps;
  const long long items = BH * splits;
  if (items >= (1LL << 31)) return ATTN_ERR_INVALID_ARG;

  DecodeParams p;
  const int dtype = BF16 ? ATTN_BF16 : ATTN_F16;
  const int page_rows = page_size < 128 ? page_size : 128;
  if (int rc = encode_bnhd(&p.tm_k, k_cache, 1, num_blocks * page_size, H, D, dtype, page_rows)) return rc;
  if (int rc = encode_bnhd(&p.tm_v, v_cache, 1, num_blocks * page_size, H, D, dtype, page_rows)) return rc;
  float* part = nullptr;
  const size_t ws_bytes = (size_t)items * (D + 2) * sizeof(float);
  if (cudaMallocAsync(reinterpret_cast<void**>(&part), ws_bytes, stream) != cudaSuccess)
    return ATTN_ERR_CUDA;
  p.q = q;
  p.part = part;
  p.status = ds->status_ptr;
  p.B = B;
  p.H = H;
  p.Nk = Nk;
  p.splits = splits;
  p.tiles_per_split = tps;
  p.n_items = (int)items;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns.load();
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.max_blocks = max_blocks;
  p.page_size = page_size;
  p.page_rows = page_rows;
  p.num_blocks = num_blocks;
  const int grid = (int)std::min<long long>(items, ds->sm_count);
  kernel<<<dim3(grid), dim3(C::kThreads), C::kSmemBytes, stream>>>(p);
  int rc = cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  if (rc == ATTN_OK) {
    attn_decode_combine_kernel<D, BF16>
        <<<dim3((unsigned)((BH + 3) / 4)), dim3(128), 0, stream>>>(part, out, lse, (int)BH, splits);
    rc = cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  if (cudaFreeAsync(part, stream) != cudaSuccess) rc = ATTN_ERR_CUDA;
  return rc;
}

// Argument checks of attn_fwd_decode_paged (nothing is enqueued on failure).
int validate_paged(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                   const int* seq_lens, const void* out, const float* lse, int B, int H, int d,
                   int num_blocks, int page_size, int max_blocks, float scale, int dtype, int splits,
                   int Lq = 1) {
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !out) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || d <= 0 || num_blocks <= 0 || page_size <= 0 || max_blocks <= 0 || splits < 0)
    return ATTN_ERR_INVALID_ARG;
  if (Lq < 1 || Lq > kMqMaxQ) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (dtype != ATTN_F16 && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  // a page is a whole number of 128-key tiles, or a tile a whole number of >= 8-row pages
  const bool page_ok = page_size < 128 ? (page_size % 8 == 0 && 128 % page_size == 0)
                                       : (page_size % 128 == 0);
  if (!page_ok) return ATTN_ERR_UNSUPPORTED;
  if ((long long)num_blocks * page_size >= (1LL << 31) || (long long)max_blocks * page_size >= (1LL << 31))
    return ATTN_ERR_INVALID_ARG;
  const unsigned long long row_bytes = (unsigned long long)H * d * 2;
  if ((unsigned long long)num_blocks * page_size * row_bytes >= (1ull << 40)) return ATTN_ERR_INVALID_ARG;
  auto misaligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) != 0; };
  if (misaligned(q, 16) || misaligned(k_cache, 16) || misaligned(v_cache, 16) || misaligned(out, 16) ||
      misaligned(block_table, 4) || misaligned(seq_lens, 4) || (lse && misaligned(lse, 4)))
    return ATTN_ERR_INVALID_ARG;
  const size_t q_bytes = (size_t)B * Lq * row_bytes;
  const size_t cache_bytes = (size_t)num_blocks * page_size * row_bytes;
  if (overlaps(out, q_bytes, q, q_bytes) || overlaps(out, q_bytes, k_cache, cache_bytes) ||
      overlaps(out, q_bytes, v_cache, cache_bytes))
    return ATTN_ERR_INVALID_ARG;
  if (lse) {
    const size_t lse_bytes = (size_t)B * H * Lq * sizeof(float);
    if (overlaps(lse, lse_bytes, out, q_bytes) || overlaps(lse, lse_bytes, q, q_bytes) ||
        overlaps(lse, lse_bytes, k_cache, cache_bytes) || overlaps(lse, lse_bytes, v_cache, cache_bytes))
      return ATTN_ERR_INVALID_ARG;
  }
  return ATTN_OK;
}

// Several query tokens per request over a paged cache: the tensor-core partial kernel,
// then the combine kernel over the key splits.
template <int D, bool BF16>
int launch_mq(DeviceState* ds, const void* q, const void* k_cache, const void* v_cache,
              const int* block_table, const int* seq_lens, void* out, float* lse, int B, int H,
              int Lq, int num_blocks, int page_size, int max_blocks, int causal, float scale,
              int splits_req, cudaStream_t stream) {
  using C = MqCfg<D>;
  auto kernel = attn_mq_partial_kernel<D, BF16>;
  const int slot = 12 + (D == 128 ? 0 : 1) + (BF16 ? 2 : 0);
  if (int rc = ensure_smem_attr(ds, slot, kernel, C::kSmemBytes)) return rc;
  const int Nk = max_blocks * page_size;  // validated < 2^31
  const int ntiles = (Nk + 127) / 128;
  const long long BH = (long long)B * H;
  int splits = splits_req > 0 ? splits_req : choose_splits(BH, ntiles, ds->sm_count);
  if (splits < 1 || splits > ntiles) return ATTN_ERR_INVALID_ARG;
  const int tps = (ntiles + splits - 1) / splits;
  splits = (ntiles + tps - 1) / tps;
  const long long items = BH * splits;
  if (items >= (1LL << 31) || items * Lq >= (1LL << 31)) return ATTN_ERR_INVALID_ARG;

  MqParams p;
  const int dtype = BF16 ? ATTN_BF16 : ATTN_F16;
  const int page_rows = page_size < 128 ? page_size : 128;
  if (int rc = encode_bnhd(&p.tm_q, q, B, Lq, H, D, dtype, kMqMaxQ)) return rc;
  if (int rc = encode_bnhd(&p.tm_k, k_cache, 1, num_blocks * page_size, H, D, dtype, page_rows)) return rc;
  if (int rc = encode_bnhd(&p.tm_v, v_cache, 1, num_blocks * page_size, H, D, dtype, page_rows)) return rc;
  float* part = nullptr;
  const size_t ws_bytes = (size_t)items * Lq * (D + 2) * sizeof(float);
  if (cudaMallocAsync(reinterpret_cast<void**>(&part), ws_bytes, stream) != cudaSuccess)
    return ATTN_ERR_CUDA;
  p.part = part;
  p.status = ds->status_ptr;
  p.B = B;
  p.H = H;
  p.Lq = Lq;
  p.Nk = Nk;
  p.causal = causal;
  p.splits = splits;
  p.tiles_per_split = tps;
  p.n_items = (int)items;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns.load();
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.max_blocks = max_blocks;
  p.page_size = page_size;
  p.page_rows = page_rows;
  p.num_blocks = num_blocks;
  const int grid = (int)std::min<long long>(items, ds->sm_count);
  kernel<<<dim3(grid), dim3(C::kThreads), C::kSmemBytes, stream>>>(p);
  int rc = cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  if (rc == ATTN_OK) {
    const long long rows = BH * Lq;
    attn_mq_combine_kernel<D, BF16><<<dim3((unsigned)((rows + 3) / 4)), dim3(128), 0, stream>>>(
        part, out, lse, B, H, Lq, splits);
    rc = cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  if (cudaFreeAsync(part, stream) != cudaSuccess) rc = ATTN_ERR_CUDA;
  return rc;
}

template <int D, bool BF16>
int launch_indexer(DeviceState* ds, const void* q, const void* kp, const float* w, const void* mask,
                   float* score, int B, int T, int H, int P, cudaStream_t stream) {
  using C = IndexerCfg<D>;
  auto kernel = attn_indexer_score_kernel<D, BF16>;
  const int slot = 16 + (D == 128 ? 0 : 1) + (BF16 ? 2 : 0);
  if (int rc = ensure_smem_attr(ds, slot, kernel, C::kSmemBytes)) return rc;
  IndexerParams p;
  const int dtype = BF16 ? ATTN_BF16 : ATTN_F16;
  if (int rc = encode_rows3d(&p.tm_q, q, B, (long long)T * H, D, dtype)) return rc;
  if (int rc = encode_rows3d(&p.tm_k, kp, B, P, D, dtype)) return rc;
  int lg = 0;
  while ((1 << lg) < H) ++lg;
  p.w = w;
  p.mask = static_cast<const uint16_t*>(mask);
  p.score = score;
  p.status = ds->status_ptr;
  p.B = B;
  p.T = T;
  p.H = H;
  p.P = P;
  p.lg_h = lg;
  p.tok_per_tile = 128 / H;
  p.mask_tma = mask != nullptr && p.tok_per_tile <= C::kMaskTokens && P % 8 == 0 &&
               reinterpret_cast<uintptr_t>(mask) % 16 == 0;
  if (p.mask_tma) {
    if (int rc = encode_mask3d(&p.tm_mask, mask, B, T, P, p.tok_per_tile)) return rc;
  } else {
    std::memset(&p.tm_mask, 0, sizeof(p.tm_mask));
  }
  p.n_ttiles = (T + p.tok_per_tile - 1) / p.tok_per_tile;
  p.n_pairs = (P + 255) / 256;
  const long long items = (long long)B * p.n_pairs * p.n_ttiles;
  if (items >= (1LL << 31)) return ATTN_ERR_INVALID_ARG;
  p.n_items = (int)items;
  p.timeout_ns = g_timeout_ns.load();
  const int grid = (int)std::min<long long>(items, ds->sm_count);
  const int per_cta = (int)((items + grid - 1) / grid);
  kernel<<<dim3(grid), dim3(C::kThreads), C::kSmemBytes, stream>>>(p, per_cta);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}


// Relative-position attention: persistent CTAs over the (batch, head, 128-query tile) units.
template <int D, bool BF16>
int launch_relpos(DeviceState* ds, const void* q, const void* k, const void* v, const void* emb, void* out,
                  float* lse, int B, int H, int Nq, int Nk, int n_emb, int R, int causal, float scale,
                  cudaStream_t stream) {
  using C = RelposCfg<D>;
  auto kernel = attn_relpos_kernel<D, BF16>;
  const int slot = 28 + (D == 128 ? 0 : 1) + (BF16 ? 2 : 0);
  if (int rc = ensure_smem_attr(ds, slot, kernel, C::kSmemBytes)) return rc;
  RelposParams p;
  const int dtype = BF16 ? ATTN_BF16 : ATTN_F16;
  if (int rc = encode_bnhd(&p.tm_q, q, B, Nq, H, D, dtype, 128)) return rc;
  if (int rc = encode_bnhd(&p.tm_k, k, B, Nk, H, D, dtype, 64)) return rc;
  if (int rc = encode_bnhd(&p.tm_v, v, B, Nk, H, D, dtype, 64)) return rc;
  if (int rc = encode_rows3d(&p.tm_e, emb, 1, n_emb, D, dtype, C::kWinRows)) return rc;
  p.out = out;
  p.lse = lse;
  p.status = ds->status_ptr;
  p.B = B;
  p.H = H;
  p.Nq = Nq;
  p.Nk = Nk;
  p.R = R;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns.load();
  p.n_qtiles = (Nq + 127) / 128;
  const long long units = (long long)B * H * p.n_qtiles;
  if (units >= (1LL << 31)) return ATTN_ERR_INVALID_ARG;
  p.n_units = (int)units;
  const int grid = (int)std::min<long long>(units, ds->sm_count);  // persistent CTAs
  kernel<<<dim3(grid), dim3(C::kThreads), C::kSmemBytes, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Backward: D = rowsum(dO o O) and a zeroed fp32 dQ accumulator, the tiled gradient
// kernel, then dQ = scale * accumulator cast to the input type.  Workspace taken
// stream-ordered from the default pool and returned on the same stream.
template <int D, bool BF16>
int launch_bwd(DeviceState* ds, const void* q, const void* k, const void* v, const void* o,
               const void* dout, const float* lse, void* dq, void* dk, void* dv, int B, int H,
               int Nq, int Nk, int causal, float scale, cudaStream_t stream) {
  using C = BwdCfg<D>;
  auto kernel = attn_bwd_kernel<D, BF16>;
  const int slot = 24 + (D == 128 ? 0 : 1) + (BF16 ? 2 : 0);
  if (int rc = ensure_smem_attr(ds, slot, kernel, C::kSmemBytes)) return rc;
  BwdParams p;
  const int dtype = BF16 ? ATTN_BF16 : ATTN_F16;
  if (int rc = encode_bnhd(&p.tm_q, q, B, Nq, H, D, dtype, 64)) return rc;
  if (int rc = encode_bnhd(&p.tm_do, dout, B, Nq, H, D, dtype, 64)) return rc;
  if (int rc = encode_bnhd(&p.tm_k, k, B, Nk, H, D, dtype)) return rc;
  if (int rc = encode_bnhd(&p.tm_v, v, B, Nk, H, D, dtype)) return rc;
  const long long rows = (long long)B * Nq * H;
  const size_t dsum_bytes = ((size_t)rows * 4 + 255) / 256 * 256;
  const size_t ws_bytes = dsum_bytes + (size_t)rows * D * 4;
  uint8_t* ws = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void**>(&ws), ws_bytes, stream) != cudaSuccess) return ATTN_ERR_CUDA;
  float* dsum = reinterpret_cast<float*>(ws);
  float* dq_acc = reinterpret_cast<float*>(ws + dsum_bytes);
  if (encode_f32_bnhd(&p.tm_dq, dq_acc, B, Nq, H, D, 64) != ATTN_OK) {
    cudaFreeAsync(ws, stream);
    return ATTN_ERR_CUDA;
  }
  p.lse = lse;
  p.dsum = dsum;
  p.dq_acc = dq_acc;
  p.dk = dk;
  p.dv = dv;
  p.status = ds->status_ptr;
  p.B = B;
  p.H = H;
  p.Nq = Nq;
  p.Nk = Nk;
  p.causal = causal;
  p.n_ktiles = (Nk + 127) / 128;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns.load();
  const long long ctas = (long long)B * H * p.n_ktiles;
  int rc = ATTN_OK;
  if (ctas >= (1LL << 31) || (rows + 3) / 4 >= (1LL << 31)) rc = ATTN_ERR_INVALID_ARG;
  if (rc == ATTN_OK) {
    attn_bwd_pre_kernel<D, BF16><<<dim3((unsigned)((rows + 3) / 4)), dim3(128), 0, stream>>>(
        o, dout, dsum, dq_acc, B, H, Nq);
    if (cudaGetLastError() != cudaSuccess) rc = ATTN_ERR_CUDA;
  }
  if (rc == ATTN_OK) {
    kernel<<<dim3((unsigned)ctas), dim3(C::kThreads), C::kSmemBytes, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) rc = ATTN_ERR_CUDA;
  }
  if (rc == ATTN_OK) {
    const long long n2 = rows * D / 2;
    attn_bwd_dq_kernel<BF16><<<dim3((unsigned)((n2 + 255) / 256)), dim3(256), 0, stream>>>(dq_acc, dq, n2, scale);
    if (cudaGetLastError() != cudaSuccess) rc = ATTN_ERR_CUDA;
  }
  if (cudaFreeAsync(ws, stream) != cudaSuccess) rc = ATTN_ERR_CUDA;
  return rc;
}

// Same kernels as launch_decode, with the partials in g_noalloc_scratch: no allocation.
template <int D, bool BF16>
int launch_decode_noalloc(DeviceState* ds, const void* q, const void* k, const void* v, void* out,
                          float* lse, int B, int H, int Nk, float scale, int splits_req,
                          cudaStream_t stream) {
  using C = DecodeCfg<D>;
  auto kernel = attn_decode_partial_kernel<D, BF16>;
  const int slot = 4 + (D == 128 ? 0 : 1) + (BF16 ? 2 : 0);
  const int ntiles = (Nk + 127) / 128;
  const long long BH = (long long)B * H;
  // automatic choice: only split counts whose partials fit the fixed array
  const long long fit = (long long)(kNoAllocScratchFloats / ((size_t)BH * (D + 2)));
  if (splits_req == 0 && fit < 1) return ATTN_ERR_INVALID_ARG;
  int splits = splits_req > 0 ? splits_req : choose_splits(BH, ntiles, ds->sm_count, fit);
  if (splits < 1 || splits > ntiles) return ATTN_ERR_INVALID_ARG;
  const int tps = (ntiles + splits - 1) / splits;
  splits = (ntiles + tps - 1) / tps;
  const long long items = BH * splits;
  if ((unsigned long long)items * (D + 2) > kNoAllocScratchFloats) return ATTN_ERR_INVALID_ARG;
  float* part = nullptr;
  if (int rc = noalloc_scratch_ptr(&part)) return rc;
  if (int rc = ensure_smem_attr(ds, slot, kernel, C::kSmemBytes)) return rc;

  DecodeParams p;
  const int dtype = BF16 ? ATTN_BF16 : ATTN_F16;
  if (int rc = encode_bnhd(&p.tm_k, k, B, Nk, H, D, dtype)) return rc;
  if (int rc = encode_bnhd(&p.tm_v, v, B, Nk, H, D, dtype)) return rc;
  p.q = q;
  p.part = part;  // every slot the combine kernel reads is written first by this call
  p.status = ds->status_ptr;
  p.B = B;
  p.H = H;
  p.Nk = Nk;
  p.splits = splits;
  p.tiles_per_split = tps;
  p.n_items = (int)items;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns.load();
  const int grid = (int)std::min<long long>(items, ds->sm_count);
  kernel<<<dim3(grid), dim3(C::kThreads), C::kSmemBytes, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  attn_decode_combine_kernel<D, BF16>
      <<<dim3((unsigned)((BH + 3) / 4)), dim3(128), 0, stream>>>(part, out, lse, (int)BH, splits);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int dispatch_prefill(DeviceState* ds, const void* q, const void* k, const void* v, void* out,
                     float* lse, int B, int H, int Nq, int Nk, int d, int causal, float scale,
                     int dtype, cudaStream_t stream) {
  const bool bf16 = dtype == ATTN_BF16;
  if (d == 128)
    return bf16 ? launch_prefill<128, true>(ds, q, k, v, out, lse, B, H, Nq, Nk, causal, scale, stream)
                : launch_prefill<128, false>(ds, q, k, v, out, lse, B, H, Nq, Nk, causal, scale, stream);
  return bf16 ? launch_prefill<64, true>(ds, q, k, v, out, lse, B, H, Nq, Nk, causal, scale, stream)
              : launch_prefill<64, false>(ds, q, k, v, out, lse, B, H, Nq, Nk, causal, scale, stream);
}

int dispatch_decode(DeviceState* ds, const void* q, const void* k, const void* v, void* out,
                    float* lse, int B, int H, int Nk, int d, float scale, int dtype, int splits,
                    cudaStream_t stream) {
  const bool bf16 = dtype == ATTN_BF16;
  if (d == 128)
    return bf16 ? launch_decode<128, true>(ds, q, k, v, out, lse, B, H, Nk, scale, splits, stream)
                : launch_decode<128, false>(ds, q, k, v, out, lse, B, H, Nk, scale, splits, stream);
  return bf16 ? launch_decode<64, true>(ds, q, k, v, out, lse, B, H, Nk, scale, splits, stream)
              : launch_decode<64, false>(ds, q, k, v, out, lse, B, H, Nk, scale, splits, stream);
}

}  // namespace

extern "C" {

int attn_fwd_prefill(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                     int H, int Nq, int Nk, int d, int causal, float scale, int dtype,
                     attn_stream_t stream) {
  if (int rc = validate(q, k, v, out, lse, B, H, Nq, Nk, d, causal, scale, dtype)) return rc;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  return dispatch_prefill(ds, q, k, v, out, lse, B, H, Nq, Nk, d, causal, scale, dtype,
                          reinterpret_cast<cudaStream_t>(stream));
}

int attn_fwd_decode(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                    int H, int Nk, int d, float scale, int dtype, int splits,
                    attn_stream_t stream) {
  if (int rc = validate(q, k, v, out, lse, B, H, 1, Nk, d, 0, scale, dtype)) return rc;
  if (splits < 0) return ATTN_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  return dispatch_decode(ds, q, k, v, out, lse, B, H, Nk, d, scale, dtype, splits,
                         reinterpret_cast<cudaStream_t>(stream));
}

int attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H,
             int Nq, int Nk, int d, int causal, float scale, int dtype, attn_stream_t stream) {
  if (int rc = validate(q, k, v, out, lse, B, H, Nq, Nk, d, causal, scale, dtype)) return rc;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  // One query row: under the bottom-right causal reading it sees every key, so
  // the causal flag changes nothing and the split-KV decode path applies.
  if (Nq == 1)
    return dispatch_decode(ds, q, k, v, out, lse, B, H, Nk, d, scale, dtype, 0,
                           reinterpret_cast<cudaStream_t>(stream));
  return dispatch_prefill(ds, q, k, v, out, lse, B, H, Nq, Nk, d, causal, scale, dtype,
                          reinterpret_cast<cudaStream_t>(stream));
}

int attn_fwd_decode_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                            int B, int H, int Nk, int d, float scale, int dtype, int splits,
                            attn_stream_t stream) {
  if (int rc = validate(q, k, v, out, lse, B, H, 1, Nk, d, 0, scale, dtype)) return rc;
  if (splits < 0) return ATTN_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == ATTN_BF16;
  if (d == 128)
    return bf16 ? launch_decode_noalloc<128, true>(ds, q, k, v, out, lse, B, H, Nk, scale, splits, st)
                : launch_decode_noalloc<128, false>(ds, q, k, v, out, lse, B, H, Nk, scale, splits, st);
  return bf16 ? launch_decode_noalloc<64, true>(ds, q, k, v, out, lse, B, H, Nk, scale, splits, st)
              : launch_decode_noalloc<64, false>(ds, q, k, v, out, lse, B, H, Nk, scale, splits, st);
}

int attn_fwd_decode_paged(const void* q, const void* k_cache, const void* v_cache,
                          const int* block_table, const int* seq_lens, void* out, float* lse, int B,
                          int H, int d, int num_blocks, int page_size, int max_blocks, float scale,
                          int dtype, int splits, attn_stream_t stream) {
  if (int rc = validate_paged(q, k_cache, v_cache, block_table, seq_lens, out, lse, B, H, d,
                              num_blocks, page_size, max_blocks, scale, dtype, splits))
    return rc;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == ATTN_BF16;
#define ATTN_PAGED_ARGS                                                                          \
  ds, q, k_cache, v_cache, block_table, seq_lens, out, lse, B, H, num_blocks, page_size, max_blocks, \
      scale, splits, st
  if (d == 128)
    return bf16 ? launch_decode_paged<128, true>(ATTN_PAGED_ARGS)
                : launch_decode_paged<128, false>(ATTN_PAGED_ARGS);
  return bf16 ? launch_decode_paged<64, true>(ATTN_PAGED_ARGS)
              : launch_decode_paged<64, false>(ATTN_PAGED_ARGS);
#undef ATTN_PAGED_ARGS
}

int attn_fwd_paged(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                   const int* seq_lens, void* out, float* lse, int B, int H, int Lq, int d,
                   int num_blocks, int page_size, int max_blocks, int causal, float scale, int dtype,
                   int splits, attn_stream_t stream) {
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (int rc = validate_paged(q, k_cache, v_cache, block_table, seq_lens, out, lse, B, H, d,
                              num_blocks, page_size, max_blocks, scale, dtype, splits, Lq))
    return rc;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == ATTN_BF16;
#define ATTN_MQ_ARGS                                                                            \
  ds, q, k_cache, v_cache, block_table, seq_lens, out, lse, B, H, Lq, num_blocks, page_size,   \
      max_blocks, causal, scale, splits, st
  if (d == 128)
    return bf16 ? launch_mq<128, true>(ATTN_MQ_ARGS) : launch_mq<128, false>(ATTN_MQ_ARGS);
  return bf16 ? launch_mq<64, true>(ATTN_MQ_ARGS) : launch_mq<64, false>(ATTN_MQ_ARGS);
#undef ATTN_MQ_ARGS
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk, int d,
             int causal, float scale, int dtype, attn_stream_t stream) {
  if (!lse || !o || !dout || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
  // q, k, v, o (as the forward's output) and the forward's own checks
  if (int rc = validate(q, k, v, o, lse, B, H, Nq, Nk, d, causal, scale, dtype)) return rc;
  auto misaligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) != 0; };
  if (misaligned(dout, 16) || misaligned(dq, 16) || misaligned(dk, 16) || misaligned(dv, 16))
    return ATTN_ERR_INVALID_ARG;
  const size_t row_bytes = (size_t)H * d * 2;
  const size_t q_bytes = (size_t)B * Nq * row_bytes, kv_bytes = (size_t)B * Nk * row_bytes;
  const void* ins[6] = {q, k, v, o, dout, lse};
  const size_t in_bytes[6] = {q_bytes, kv_bytes, kv_bytes, q_bytes, q_bytes, (size_t)B * H * Nq * 4};
  void* outs[3] = {dq, dk, dv};
  const size_t out_bytes[3] = {q_bytes, kv_bytes, kv_bytes};
  for (int a = 0; a < 3; ++a) {
    for (int c = 0; c < 6; ++c)
      if (overlaps(outs[a], out_bytes[a], ins[c], in_bytes[c])) return ATTN_ERR_INVALID_ARG;
    for (int c = a + 1; c < 3; ++c)
      if (overlaps(outs[a], out_bytes[a], outs[c], out_bytes[c])) return ATTN_ERR_INVALID_ARG;
  }
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == ATTN_BF16;
#define ATTN_BWD_ARGS ds, q, k, v, o, dout, lse, dq, dk, dv, B, H, Nq, Nk, causal, scale, st
  if (d == 128)
    return bf16 ? launch_bwd<128, true>(ATTN_BWD_ARGS) : launch_bwd<128, false>(ATTN_BWD_ARGS);
  return bf16 ? launch_bwd<64, true>(ATTN_BWD_ARGS) : launch_bwd<64, false>(ATTN_BWD_ARGS);
#undef ATTN_BWD_ARGS
}

int attn_fwd_relpos(const void* q, const void* k, const void* v, const void* emb, void* out, float* lse,
                    int B, int H, int Nq, int Nk, int d, int n_emb, int R, int causal, float scale,
                    int dtype, attn_stream_t stream) {
  if (int rc = validate(q, k, v, out, lse, B, H, Nq, Nk, d, causal, scale, dtype)) return rc;
  if (!emb || R < 0 || n_emb < 2 * (long long)R + 1) return ATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(emb) % 16 != 0) return ATTN_ERR_INVALID_ARG;
  if ((unsigned long long)n_emb * d * 2 >= (1ull << 40)) return ATTN_ERR_INVALID_ARG;
  const size_t q_bytes = (size_t)B * Nq * H * d * 2;
  if (overlaps(out, q_bytes, emb, (size_t)n_emb * d * 2) ||
      (lse && overlaps(lse, (size_t)B * H * Nq * 4, emb, (size_t)n_emb * d * 2)))
    return ATTN_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == ATTN_BF16;
#define ATTN_RELPOS_ARGS ds, q, k, v, emb, out, lse, B, H, Nq, Nk, n_emb, R, causal, scale, st
  if (d == 128)
    return bf16 ? launch_relpos<128, true>(ATTN_RELPOS_ARGS) : launch_relpos<128, false>(ATTN_RELPOS_ARGS);
  return bf16 ? launch_relpos<64, true>(ATTN_RELPOS_ARGS) : launch_relpos<64, false>(ATTN_RELPOS_ARGS);
#undef ATTN_RELPOS_ARGS
}

int attn_indexer_score(const void* q, const void* kp, const float* w, const void* mask, float* score,
                       int B, int T, int H, int P, int d, int dtype, attn_stream_t stream) {
  if (!q || !kp || !w || !score) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || T <= 0 || H <= 0 || P <= 0 || d <= 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (dtype != ATTN_F16 && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  if (H > 128 || (H & (H - 1)) != 0) return ATTN_ERR_UNSUPPORTED;
  auto misaligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) != 0; };
  if (misaligned(q, 16) || misaligned(kp, 16) || misaligned(w, 4) || misaligned(score, 4) ||
      (mask && misaligned(mask, 2)))
    return ATTN_ERR_INVALID_ARG;
  const unsigned long long q_bytes = (unsigned long long)B * T * H * d * 2;
  const unsigned long long k_bytes = (unsigned long long)B * P * d * 2;
  const unsigned long long s_bytes = (unsigned long long)B * T * P * 4;
  if ((unsigned long long)T * H * d * 2 >= (1ull << 40) || (unsigned long long)P * d * 2 >= (1ull << 40))
    return ATTN_ERR_INVALID_ARG;
  if (overlaps(score, s_bytes, q, q_bytes) || overlaps(score, s_bytes, kp, k_bytes) ||
      overlaps(score, s_bytes, w, (size_t)B * T * H * 4) ||
      (mask && overlaps(score, s_bytes, mask, (size_t)B * T * P * 2)))
    return ATTN_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == ATTN_BF16;
  if (d == 128)
    return bf16 ? launch_indexer<128, true>(ds, q, kp, w, mask, score, B, T, H, P, st)
                : launch_indexer<128, false>(ds, q, kp, w, mask, score, B, T, H, P, st);
  return bf16 ? launch_indexer<64, true>(ds, q, kp, w, mask, score, B, T, H, P, st)
              : launch_indexer<64, false>(ds, q, kp, w, mask, score, B, T, H, P, st);
}

int attn_topk(const float* score, int R, int P, int k, int* idx, attn_stream_t stream) {
  if (!score || !idx) return ATTN_ERR_INVALID_ARG;
  if (R <= 0 || P <= 0 || k <= 0 || k > kTopkMaxK) return ATTN_ERR_INVALID_ARG;
  auto misaligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) != 0; };
  if (misaligned(score, 4) || misaligned(idx, 4)) return ATTN_ERR_INVALID_ARG;
  if (overlaps(idx, (size_t)R * k * 4, score, (size_t)R * P * 4)) return ATTN_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int kp2 = 1;
  while (kp2 < k) kp2 <<= 1;
  const bool cached = P <= kTopkCache;
  const size_t smem = (size_t)(296 + 2 * kp2 + (cached ? P : 0)) * 4;
  if (cached) {
    if (int rc = ensure_smem_attr(ds, 20, attn_topk_kernel<true>, (int)((296 + 2 * kTopkMaxK + kTopkCache) * 4)))
      return rc;
    attn_topk_kernel<true><<<dim3(R), dim3(kTopkThreads), smem, st>>>(score, R, P, k, idx);
  } else {
    if (int rc = ensure_smem_attr(ds, 21, attn_topk_kernel<false>, (int)((296 + 2 * kTopkMaxK) * 4)))
      return rc;
    attn_topk_kernel<false><<<dim3(R), dim3(kTopkThreads), smem, st>>>(score, R, P, k, idx);
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_get_status(attn_stream_t stream) {
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  int value = 0;
  if (cudaMemcpy(&value, ds->status_ptr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return ATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(ds->status_ptr, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return value;
}

const char* attn_error_string(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK: success";
    case ATTN_ERR_INVALID_ARG:
      return "ATTN_ERR_INVALID_ARG: null pointer, non-positive size, misaligned or overlapping "
             "buffer, non-finite scale or size beyond a limit";
    case ATTN_ERR_UNSUPPORTED:
      return "ATTN_ERR_UNSUPPORTED: head_dim must be 64 or 128, dtype f16/bf16, device sm_100";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA: a CUDA runtime or driver call failed";
    case ATTN_ERR_TIMEOUT:
      return "ATTN_ERR_TIMEOUT: a bounded device-side pipeline wait expired; outputs undefined";
    case ATTN_ERR_RANGE:
      return "ATTN_ERR_RANGE: a bf16 V value of magnitude >= 65536 (or inf/NaN) has no fp16 value; "
             "outputs undefined";
    default: return "unknown attn status code";
  }
}

int attn_version(void) { return kVersion; }


int attn_debug_set(int inject, unsigned long long wait_timeout_ns) {
  g_inject.store(inject);
  g_timeout_ns.store(wait_timeout_ns ? wait_timeout_ns : kDefaultTimeoutNs);
  return ATTN_OK;
}

}  // extern "C"
