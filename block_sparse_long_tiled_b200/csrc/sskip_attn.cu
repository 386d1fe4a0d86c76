// sskip_attn.cu -- the C ABI of libsskip_attn.so (declared in
// include/sskip_attn.h): argument validation, TMA descriptor set-up and the
// launches of the sm_100a kernels.  One translation unit, so the device status
// word is shared by every kernel without relocatable device code.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>
#include <algorithm>
#include <vector>

#include "../../include/sskip_attn.h"
#include "decode_sm100.cuh"
#include "permute_sm100.cuh"
#include "prefill_sm100.cuh"

#define SSKIP_API extern "C" __attribute__((visibility("default")))

namespace sskip {

// A kernel that waits on an mbarrier nothing will ever complete: its bounded
// wait must run out, latch SSKIP_ERR_TIMEOUT and return.
__global__ void watchdog_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, (volatile int*)&abort_flag, limit_ns);
}

namespace {

constexpr int kVersion = 100;  // 0.1.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D bf16 map over a [planes, rows, d] tensor, box {64, box_rows, 1},
// 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* map, const void* base, int d, int rows, long long planes, int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)planes};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * 2 * (cuuint64_t)rows};
  cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}

// Raise a kernel's dynamic shared memory limit once per (kernel, device).
cudaError_t ensure_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  const std::pair<const void*, int> key(kernel, current_device());
  std::lock_guard<std::mutex> lk(mu);
  if (done.count(key)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.insert(key);
  return e;
}

template <int D, int BR, int BC, bool CAUSAL, bool EXT>
int launch_prefill_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const PrefillParams& p, cudaStream_t st) {
  auto kernel = prefill_kernel<D, BR, BC, CAUSAL, EXT>;
  const int smem = PrefillCfg<D, BC>::kAlloc;
  if (ensure_smem(reinterpret_cast<const void*>(kernel), smem) != cudaSuccess)
    return SSKIP_ERR_CUDA;
  const long long grid = (long long)p.B * p.Hq * p.n_units;
  kernel<<<(unsigned)grid, kPfThreads, smem, st>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? SSKIP_OK : SSKIP_ERR_CUDA;
}

template <int D, int G>
int launch_decode(const DecodeParams& p, cudaStream_t st) {
  auto kernel = p.tile_crit ? decode_split_kernel<D, G, true> : decode_split_kernel<D, G, false>;
  const int smem = DecodeSmem<D, G>::kTotal;
  if (ensure_smem(reinterpret_cast<const void*>(kernel), smem) != cudaSuccess)
    return SSKIP_ERR_CUDA;
  dim3 grid(p.S, p.Hkv, p.B);
  kernel<<<grid, kDecThreads, smem, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return SSKIP_ERR_CUDA;
  decode_combine_kernel<D><<<(unsigned)(p.B * p.Hq), 128, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SSKIP_OK : SSKIP_ERR_CUDA;
}

template <int D, int BR, int BC, bool CAUSAL>
int launch_prefill(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                   const PrefillParams& p, cudaStream_t st) {
  const bool ext = p.slice_vote || p.slice_mask || p.tile_crit || p.n_counts == 4;
  return ext ? launch_prefill_t<D, BR, BC, CAUSAL, true>(mq, mk, mv, p, st)
             : launch_prefill_t<D, BR, BC, CAUSAL, false>(mq, mk, mv, p, st);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace
}  // namespace sskip

using namespace sskip;

SSKIP_API int sskip_version(void) { return kVersion; }

SSKIP_API const char* sskip_status_string(int status) {
  switch (status) {
    case SSKIP_OK: return "ok";
    case SSKIP_ERR_INVALID_ARG: return "invalid argument";
    case SSKIP_ERR_UNSUPPORTED: return "unsupported configuration";
    case SSKIP_ERR_CUDA: return "CUDA error";
    case SSKIP_ERR_TIMEOUT: return "device-side wait timed out";
    case SSKIP_ERR_DEVICE_CHECK: return "device-side index check failed (debug build)";
    default: return "unknown status";
  }
}

SSKIP_API int sskip_device_supported(int device) {
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return SSKIP_ERR_CUDA;
  return (prop.major == 10 && prop.minor == 0) ? SSKIP_OK : SSKIP_ERR_UNSUPPORTED;
}

namespace sskip {
namespace {

// The synchronous argument checks of a prefill call (pointers, alignment,
// shapes, scale and factor, supported tile sizes).
int prefill_check(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  int B, int Hq, int Hkv, int L, int d, float sm_scale,
                  float threshold_scale_factor, int Br, int Bc, int vote_rows,
                  const unsigned long long* counts, const float* tile_crit) {
  if (!q || !k || !v || !o || !lse) return SSKIP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(counts) & 7u) ||
      (reinterpret_cast<uintptr_t>(tile_crit) & 3u))
    return SSKIP_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || Hq % Hkv != 0) return SSKIP_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SSKIP_ERR_INVALID_ARG;
  if (!(threshold_scale_factor >= 0.f) || !std::isfinite(threshold_scale_factor))
    return SSKIP_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SSKIP_ERR_UNSUPPORTED;
  if (!((Br == 64 && Bc == 64) || (Br == 128 && Bc == 128))) return SSKIP_ERR_UNSUPPORTED;
  if (vote_rows != Br && vote_rows != 32) return SSKIP_ERR_UNSUPPORTED;
  const long long n_units = (L + kPfUnitRows - 1) / kPfUnitRows;
  if ((long long)B * Hq * n_units >= (1ll << 31) || (long long)B * Hq >= (1ll << 31))
    return SSKIP_ERR_UNSUPPORTED;
  return SSKIP_OK;
}

int prefill_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                 int Hkv, int L, int d, int causal, float sm_scale, float threshold_scale_factor,
                 int Br, int Bc, int vote_rows, unsigned long long* counts, int n_counts,
                 uint8_t* tile_state, uint8_t* slice_mask, float* tile_crit, void* stream,
                 bool zero_counts = true) {
  const int rc = prefill_check(q, k, v, o, lse, B, Hq, Hkv, L, d, sm_scale,
                               threshold_scale_factor, Br, Bc, vote_rows, counts, tile_crit);
  if (rc != SSKIP_OK) return rc;
  const long long n_units = (L + kPfUnitRows - 1) / kPfUnitRows;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, d, L, (long long)B * Hq, 128) ||
      !make_map(&mk, k, d, L, (long long)B * Hkv, Bc) ||
      !make_map(&mv, v, d, L, (long long)B * Hkv, Bc))
    return SSKIP_ERR_CUDA;

  PrefillParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.counts = counts;
  p.n_counts = n_counts;
  p.tile_state = tile_state;
  p.slice_mask = slice_mask;
  p.slice_vote = vote_rows != Br;
  p.tile_crit = tile_crit;
  p.ln_L = (float)std::log((double)L);
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.L = L; p.G = Hq / Hkv;
  p.n_q = (L + Br - 1) / Br;
  p.n_k = (L + Bc - 1) / Bc;
  p.n_units = (int)n_units;
  p.scale_log2 = (float)((double)sm_scale * 1.4426950408889634);
  p.t_positive = threshold_scale_factor > 0.f;
  p.log2_t = p.t_positive ? (float)std::log2((double)threshold_scale_factor / (double)L)
                          : -INFINITY;

  if (counts && zero_counts &&
      cudaMemsetAsync(counts, 0, (size_t)n_counts * sizeof(unsigned long long), st) != cudaSuccess)
    return SSKIP_ERR_CUDA;
  if (tile_state &&
      cudaMemsetAsync(tile_state, 0, (size_t)B * Hq * p.n_q * p.n_k, st) != cudaSuccess)
    return SSKIP_ERR_CUDA;
  if (slice_mask &&
      cudaMemsetAsync(slice_mask, 0, (size_t)B * Hq * p.n_q * p.n_k, st) != cudaSuccess)
    return SSKIP_ERR_CUDA;
  // 0xFF bytes are a NaN: tiles a call never visits stay NaN.
  if (tile_crit &&
      cudaMemsetAsync(tile_crit, 0xFF, (size_t)B * Hq * p.n_q * p.n_k * 4, st) != cudaSuccess)
    return SSKIP_ERR_CUDA;

  const bool c = causal != 0;
  if (d == 128 && Br == 128) return c ? launch_prefill<128, 128, 128, true>(mq, mk, mv, p, st)
                                      : launch_prefill<128, 128, 128, false>(mq, mk, mv, p, st);
  if (d == 64 && Br == 128) return c ? launch_prefill<64, 128, 128, true>(mq, mk, mv, p, st)
                                     : launch_prefill<64, 128, 128, false>(mq, mk, mv, p, st);
  if (d == 128 && Br == 64) return c ? launch_prefill<128, 64, 64, true>(mq, mk, mv, p, st)
                                     : launch_prefill<128, 64, 64, false>(mq, mk, mv, p, st);
  return c ? launch_prefill<64, 64, 64, true>(mq, mk, mv, p, st)
           : launch_prefill<64, 64, 64, false>(mq, mk, mv, p, st);
}

}  // namespace
}  // namespace sskip

SSKIP_API int sskip_attn_prefill_ex(const void* q, const void* k, const void* v, void* o,
                                    float* lse, int B, int Hq, int Hkv, int L, int d, int causal,
                                    float sm_scale, float threshold_scale_factor, int Br, int Bc,
                                    unsigned long long* skip_count, uint8_t* tile_state,
                                    void* stream) {
  return prefill_impl(q, k, v, o, lse, B, Hq, Hkv, L, d, causal, sm_scale, threshold_scale_factor,
                      Br, Bc, Br, skip_count, 2, tile_state, nullptr, nullptr, stream);
}

SSKIP_API int sskip_attn_prefill_vote(const void* q, const void* k, const void* v, void* o,
                                      float* lse, int B, int Hq, int Hkv, int L, int d, int causal,
                                      float sm_scale, float threshold_scale_factor, int Br, int Bc,
                                      int vote_rows, unsigned long long* counts,
                                      uint8_t* tile_state, uint8_t* slice_mask, float* tile_crit,
                                      void* stream) {
  return prefill_impl(q, k, v, o, lse, B, Hq, Hkv, L, d, causal, sm_scale, threshold_scale_factor,
                      Br, Bc, vote_rows, counts, 4, tile_state, slice_mask, tile_crit, stream);
}

SSKIP_API int sskip_attn_prefill(const void* q, const void* k, const void* v, void* o, float* lse,
                                 int B, int Hq, int Hkv, int L, int d, int causal, float sm_scale,
                                 float threshold_scale_factor, int Br, int Bc,
                                 unsigned long long* skip_count, void* stream) {
  return sskip_attn_prefill_ex(q, k, v, o, lse, B, Hq, Hkv, L, d, causal, sm_scale,
                               threshold_scale_factor, Br, Bc, skip_count, nullptr, stream);
}

SSKIP_API size_t sskip_attn_decode_workspace_size(int B, int Hq, int d, int num_splits) {
  if (B < 1 || Hq < 1 || d < 1 || num_splits < 1) return 0;
  const size_t rows = (size_t)B * Hq * num_splits;
  return align256(rows * d * sizeof(float)) + align256(rows * sizeof(float));
}

namespace sskip {
namespace {

int decode_impl(const void* q, const void* kcache, const void* vcache, const int* seqlens, void* o,
                float* lse, int B, int Hq, int Hkv, int Lmax, int d, float sm_scale,
                float threshold_scale_factor, int Bc, int num_splits, void* workspace,
                size_t workspace_bytes, unsigned long long* skip_count, uint8_t* tile_state,
                float* tile_crit, void* stream) {
  if (!q || !kcache || !vcache || !seqlens || !o || !lse || !workspace)
    return SSKIP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(skip_count) & 7u) || (reinterpret_cast<uintptr_t>(tile_crit) & 3u))
    return SSKIP_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Lmax < 1 || Hq % Hkv != 0 || num_splits < 1)
    return SSKIP_ERR_INVALID_ARG;
  if (B > 65535 || Hkv > 65535) return SSKIP_ERR_UNSUPPORTED;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SSKIP_ERR_INVALID_ARG;
  if (!(threshold_scale_factor >= 0.f) || !std::isfinite(threshold_scale_factor))
    return SSKIP_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (d != 64 && d != 128) return SSKIP_ERR_UNSUPPORTED;
  if (Bc != kDecBc || num_splits > 64) return SSKIP_ERR_UNSUPPORTED;
  if (G != 1 && G != 2 && G != 4 && G != 8) return SSKIP_ERR_UNSUPPORTED;
  if (workspace_bytes < sskip_attn_decode_workspace_size(B, Hq, d, num_splits))
    return SSKIP_ERR_INVALID_ARG;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t rows = (size_t)B * Hq * num_splits;
  DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kc = static_cast<const __nv_bfloat16*>(kcache);
  p.vc = static_cast<const __nv_bfloat16*>(vcache);
  p.seqlens = seqlens;
  p.o_part = static_cast<float*>(workspace);
  p.lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(rows * d * 4));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.counts = skip_count;
  p.tile_state = tile_state;
  p.tile_crit = tile_crit;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lmax = Lmax; p.S = num_splits;
  p.n_k_max = (Lmax + kDecBc - 1) / kDecBc;
  p.scale_log2 = (float)((double)sm_scale * 1.4426950408889634);
  p.tsf = threshold_scale_factor;

  if (skip_count && cudaMemsetAsync(skip_count, 0, 2 * sizeof(unsigned long long), st) != cudaSuccess)
    return SSKIP_ERR_CUDA;
  if (tile_state &&
      cudaMemsetAsync(tile_state, 0, (size_t)B * Hkv * p.n_k_max, st) != cudaSuccess)
    return SSKIP_ERR_CUDA;
  // 0xFF bytes are a NaN: tiles a call never visits stay NaN.
  if (tile_crit &&
      cudaMemsetAsync(tile_crit, 0xFF, (size_t)B * Hkv * p.n_k_max * 4, st) != cudaSuccess)
    return SSKIP_ERR_CUDA;

  if (d == 128) {
    switch (G) {
      case 1: return launch_decode<128, 1>(p, st);
      case 2: return launch_decode<128, 2>(p, st);
      case 4: return launch_decode<128, 4>(p, st);
      default: return launch_decode<128, 8>(p, st);
    }
  }
  switch (G) {
    case 1: return launch_decode<64, 1>(p, st);
    case 2: return launch_decode<64, 2>(p, st);
    case 4: return launch_decode<64, 4>(p, st);
    default: return launch_decode<64, 8>(p, st);
  }
}

}  // namespace
}  // namespace sskip

SSKIP_API int sskip_attn_decode_ex(const void* q, const void* kcache, const void* vcache,
                                   const int* seqlens, void* o, float* lse, int B, int Hq, int Hkv,
                                   int Lmax, int d, float sm_scale, float threshold_scale_factor,
                                   int Bc, int num_splits, void* workspace, size_t workspace_bytes,
                                   unsigned long long* skip_count, uint8_t* tile_state,
                                   void* stream) {
  return decode_impl(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, Lmax, d, sm_scale,
                     threshold_scale_factor, Bc, num_splits, workspace, workspace_bytes,
                     skip_count, tile_state, nullptr, stream);
}

SSKIP_API int sskip_attn_decode_crit(const void* q, const void* kcache, const void* vcache,
                                     const int* seqlens, void* o, float* lse, int B, int Hq,
                                     int Hkv, int Lmax, int d, float sm_scale,
                                     float threshold_scale_factor, int Bc, int num_splits,
                                     void* workspace, size_t workspace_bytes,
                                     unsigned long long* skip_count, uint8_t* tile_state,
                                     float* tile_crit, void* stream) {
  return decode_impl(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, Lmax, d, sm_scale,
                     threshold_scale_factor, Bc, num_splits, workspace, workspace_bytes,
                     skip_count, tile_state, tile_crit, stream);
}

SSKIP_API int sskip_attn_decode(const void* q, const void* kcache, const void* vcache,
                                const int* seqlens, void* o, float* lse, int B, int Hq, int Hkv,
                                int Lmax, int d, float sm_scale, float threshold_scale_factor,
                                int Bc, int num_splits, void* workspace, size_t workspace_bytes,
                                unsigned long long* skip_count, void* stream) {
  return sskip_attn_decode_ex(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, Lmax, d, sm_scale,
                              threshold_scale_factor, Bc, num_splits, workspace, workspace_bytes,
                              skip_count, nullptr, stream);
}

SSKIP_API int sskip_get_status(void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return SSKIP_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return SSKIP_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return SSKIP_ERR_CUDA;
  }
  return v;
}

SSKIP_API int sskip_selftest_watchdog(unsigned int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 2000000u) return SSKIP_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  watchdog_selftest_kernel<<<1, 32, 0, st>>>((uint64_t)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? SSKIP_OK : SSKIP_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Decode without any allocation by the caller.
//
// Some callers cannot call cudaMalloc at all -- embedded runtimes without a
// device allocator, plugins whose host framework owns every device
// allocation, serving loops that forbid allocation after start-up -- yet the
// split-KV decode needs scratch for its per-split partial results.  For them the scratch lives in one fixed
// device array of this library.  Every GPU that loads the library reserves it
// for the life of the process.
namespace sskip {
namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[SSKIP_DECODE_NOALLOC_SCRATCH_BYTES];

// The host-side name g_decode_scratch is only a stand-in for the device array;
// its device address is looked up once per device, with that device current.
void* decode_scratch_on_current_device() {
  static std::mutex mu;
  static void* addr[64] = {};
  const int dev = current_device();
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace
}  // namespace sskip

SSKIP_API int sskip_attn_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                                        const int* seqlens, void* o, float* lse, int B, int Hq,
                                        int Hkv, int Lmax, int d, float sm_scale,
                                        float threshold_scale_factor, int Bc, int num_splits,
                                        unsigned long long* skip_count, void* stream) {
  const size_t need = sskip_attn_decode_workspace_size(B, Hq, d, num_splits);
  if (need == 0) return SSKIP_ERR_INVALID_ARG;
  if (need > (size_t)SSKIP_DECODE_NOALLOC_SCRATCH_BYTES) return SSKIP_ERR_UNSUPPORTED;
  void* scratch = decode_scratch_on_current_device();
  if (!scratch) return SSKIP_ERR_CUDA;
  return sskip_attn_decode_ex(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, Lmax, d, sm_scale,
                              threshold_scale_factor, Bc, num_splits, scratch,
                              (size_t)SSKIP_DECODE_NOALLOC_SCRATCH_BYTES, skip_count, nullptr,
                              stream);
}

// ---------------------------------------------------------------------------
// Threshold calibration: choose the factor that skips a target share of tiles.
//
// While t < 1 no passing row can raise its running maximum, so the running
// maximum is the prefix maximum of the local maxima whatever was skipped and a
// tile is skipped exactly when ln(factor) exceeds its critical value
// c = max_rows (m_local - m_run) + ln L.  The skip count is therefore the
// number of critical values below ln(factor), and the factor for a target
// count k lies just above the k-th smallest critical value.  The factor is
// placed halfway (in ln) between that value and the next larger one, away
// from both decision boundaries.
SSKIP_API int sskip_calibrate_factor(const float* tile_crit, size_t n, double target_ratio,
                                     double max_factor, double* factor, double* achieved_ratio,
                                     long long* visited_out) {
  if (!tile_crit || !factor || !(target_ratio >= 0.0) || !(target_ratio <= 1.0))
    return SSKIP_ERR_INVALID_ARG;
  std::vector<float> c;
  c.reserve(n);
  long long visited = 0;
  for (size_t i = 0; i < n; ++i) {
    const float x = tile_crit[i];
    if (x != x) continue;  // not visited
    ++visited;
    if (x < INFINITY) c.push_back(x);
  }
  if (visited_out) *visited_out = visited;
  if (visited == 0) return SSKIP_ERR_INVALID_ARG;
  const long long k = std::min<long long>(
      visited, std::max<long long>(0, (long long)std::ceil(target_ratio * (double)visited - 1e-9)));
  const double ln_max = max_factor > 0.0 ? std::log(max_factor) : INFINITY;
  if (k == 0) {
    *factor = 0.0;  // factor 0 skips nothing
    if (achieved_ratio) *achieved_ratio = 0.0;
    return SSKIP_OK;
  }
  if (k > (long long)c.size()) return SSKIP_ERR_UNSUPPORTED;
  std::nth_element(c.begin(), c.begin() + (k - 1), c.end());
  const double ck = c[k - 1];
  double cn = INFINITY;  // next larger critical value
  for (size_t i = (size_t)k; i < c.size(); ++i)
    if (c[i] > ck && c[i] < cn) cn = c[i];
  if (!(ck < ln_max)) return SSKIP_ERR_UNSUPPORTED;  // would need t >= 1
  const double hi = std::min(cn, ln_max);
  double ln_f;
  if (std::isinf(ck)) ln_f = std::isinf(hi) ? 0.0 : hi - 1.0;  // ck = -inf: any factor > 0
  else ln_f = std::isinf(hi) ? ck + 1.0 : 0.5 * (ck + hi);
  *factor = std::exp(ln_f);
  if (achieved_ratio) {
    long long below = 0;
    for (float x : c) below += (double)x < ln_f;
    *achieved_ratio = (double)below / (double)visited;
  }
  return SSKIP_OK;
}

// ---------------------------------------------------------------------------
// Token reordering (SpargeAttn article, "Hilbert 曲线置换").
namespace sskip {
namespace {

// Position of a 3-D point on the Hilbert curve of side 2^bits, by John
// Skilling's method ("Programming the Hilbert curve", AIP Conf. Proc. 707,
// 2004): the axes are turned into the transposed index by undoing the curve's
// reflections and exchanges from the top bit down plus a Gray code, and the
// transposed index is read out bit plane by bit plane.
uint64_t hilbert3(uint32_t a0, uint32_t a1, uint32_t a2, int bits) {
  uint32_t ax[3] = {a0, a1, a2};
  for (uint32_t q = 1u << (bits - 1); q > 1; q >>= 1) {
    const uint32_t low = q - 1;
    for (int d = 0; d < 3; ++d) {
      if (ax[d] & q) {
        ax[0] ^= low;
      } else {
        const uint32_t sw = (ax[0] ^ ax[d]) & low;
        ax[0] ^= sw;
        ax[d] ^= sw;
      }
    }
  }
  ax[1] ^= ax[0];
  ax[2] ^= ax[1];
  uint32_t flip = 0;
  for (uint32_t q = 1u << (bits - 1); q > 1; q >>= 1)
    if (ax[2] & q) flip ^= q - 1;
  for (int d = 0; d < 3; ++d) ax[d] ^= flip;
  uint64_t h = 0;
  for (int bit = bits - 1; bit >= 0; --bit)
    for (int d = 0; d < 3; ++d) h = (h << 1) | ((ax[d] >> bit) & 1u);
  return h;
}

}  // namespace
}  // namespace sskip

SSKIP_API int sskip_hilbert3d_order(int T, int H, int W, int L, int32_t* perm) {
  if (!perm || T < 1 || H < 1 || W < 1 || L < 1 || (long long)T * H * W < L)
    return SSKIP_ERR_INVALID_ARG;
  int bits = 1;
  while ((1 << bits) < std::max(T, std::max(H, W))) ++bits;
  if (bits > 20) return SSKIP_ERR_UNSUPPORTED;
  std::vector<std::pair<uint64_t, int32_t>> key(L);
  for (int i = 0; i < L; ++i) {
    const int t = i / (H * W), h = (i / W) % H, w = i % W;  // t-major raster
    key[i] = {hilbert3((uint32_t)t, (uint32_t)h, (uint32_t)w, bits), i};
  }
  std::sort(key.begin(), key.end());  // keys are distinct: a bijection of the cube
  for (int s = 0; s < L; ++s) perm[s] = key[s].second;
  return SSKIP_OK;
}

SSKIP_API int sskip_permute_rows(const void* src, void* dst, const int32_t* idx, long long n_mats,
                                 int L, int row_bytes, int scatter, void* stream) {
  if (!src || !dst || !idx || src == dst || n_mats < 1 || L < 1 || row_bytes < 4 ||
      row_bytes % 4 != 0 || (reinterpret_cast<uintptr_t>(idx) & 3u))
    return SSKIP_ERR_INVALID_ARG;
  const bool v16 = row_bytes % 16 == 0 && aligned16(src) && aligned16(dst);
  if (!v16 && ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 3u))
    return SSKIP_ERR_INVALID_ARG;
  const int cpr = row_bytes / (v16 ? 16 : 4);
  const long long total = n_mats * (long long)L * cpr;
  int sms = 148;
  {
    int dev = current_device();
    if (dev >= 0) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const long long want = (total + 255) / 256;
  const unsigned grid = (unsigned)std::max<long long>(1, std::min<long long>(want, (long long)sms * 8));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (v16)
    permute_rows_kernel<uint4><<<grid, 256, 0, st>>>(static_cast<const uint4*>(src),
                                                     static_cast<uint4*>(dst), idx, n_mats, L, cpr,
                                                     scatter != 0);
  else
    permute_rows_kernel<uint32_t><<<grid, 256, 0, st>>>(static_cast<const uint32_t*>(src),
                                                         static_cast<uint32_t*>(dst), idx, n_mats,
                                                         L, cpr, scatter != 0);
  return cudaGetLastError() == cudaSuccess ? SSKIP_OK : SSKIP_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// One serving step with a factor per phase (TensorRT-LLM article, "实战演练":
// threshold_scale_factor may be one number or a {prefill, decode} pair).
SSKIP_API int sskip_attn_step(const void* q, const void* k, const void* v, void* o, float* lse,
                              int Bp, int L, int causal, int Br, int Bc,
                              unsigned long long* prefill_count, const void* dq,
                              const void* kcache, const void* vcache, const int* seqlens,
                              void* dout, float* dlse, int Bd, int Lmax, int num_splits,
                              void* workspace, size_t workspace_bytes,
                              unsigned long long* decode_count, int Hq, int Hkv, int d,
                              float sm_scale, float tsf_prefill, float tsf_decode, void* stream) {
  if (Bp < 0 || Bd < 0 || Bp + Bd == 0) return SSKIP_ERR_INVALID_ARG;
  if (Bp > 0) {
    const int rc = sskip_attn_prefill_ex(q, k, v, o, lse, Bp, Hq, Hkv, L, d, causal, sm_scale,
                                         tsf_prefill, Br, Bc, prefill_count, nullptr, stream);
    if (rc != SSKIP_OK) return rc;
  }
  if (Bd > 0)
    return sskip_attn_decode_ex(dq, kcache, vcache, seqlens, dout, dlse, Bd, Hq, Hkv, Lmax, d,
                                sm_scale, tsf_decode, kDecBc, num_splits, workspace,
                                workspace_bytes, decode_count, nullptr, stream);
  return SSKIP_OK;
}

// ---------------------------------------------------------------------------
// Prefill from and to host memory, with the copies overlapped with the
// kernels: the work is cut into groups of kv heads (each group's query heads,
// keys, values, outputs and lse rows are contiguous in the [B, H, L, ...]
// layouts), and group i's copy in, group i-1's prefill and group i-2's copy
// out run at the same time on three streams.
namespace sskip {
namespace {

struct CopyStreams {
  cudaStream_t in = nullptr, out = nullptr;
};

// Two non-blocking copy streams per device, created on first use and kept
// for the life of the process.
int copy_streams(CopyStreams* cs) {
  static std::mutex mu;
  static CopyStreams per_dev[64];
  const int dev = current_device();
  if (dev < 0 || dev >= 64) return SSKIP_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  CopyStreams& c = per_dev[dev];
  if (!c.in && cudaStreamCreateWithFlags(&c.in, cudaStreamNonBlocking) != cudaSuccess)
    return SSKIP_ERR_CUDA;
  if (!c.out && cudaStreamCreateWithFlags(&c.out, cudaStreamNonBlocking) != cudaSuccess)
    return SSKIP_ERR_CUDA;
  *cs = c;
  return SSKIP_OK;
}

}  // namespace
}  // namespace sskip

SSKIP_API int sskip_attn_prefill_host(const void* q_h, const void* k_h, const void* v_h, void* o_h,
                                      float* lse_h, void* q_d, void* k_d, void* v_d, void* o_d,
                                      float* lse_d, int B, int Hq, int Hkv, int L, int d,
                                      int causal, float sm_scale, float threshold_scale_factor,
                                      int Br, int Bc, int kv_per_chunk,
                                      unsigned long long* skip_count, void* stream) {
  if (!q_h || !k_h || !v_h || !o_h || !lse_h || kv_per_chunk < 0) return SSKIP_ERR_INVALID_ARG;
  // Every check a chunk's prefill would make, before the first copy: the
  // chunks' offsets keep the base pointers' alignment (a head's [L, d] bf16
  // matrix is a multiple of 128 bytes, its lse row of 4).
  int rc = prefill_check(q_d, k_d, v_d, o_d, lse_d, B, Hq, Hkv, L, d, sm_scale,
                         threshold_scale_factor, Br, Bc, Br, skip_count, nullptr);
  if (rc != SSKIP_OK) return rc;
  const int G = Hq / Hkv;
  const int n_units = (L + kPfUnitRows - 1) / kPfUnitRows;
  int kc = kv_per_chunk;
  if (kc == 0) {  // the smallest group that still fills one wave of a 148-SM part
    const int per_kv = G * n_units;
    kc = std::max(1, (148 + per_kv - 1) / per_kv);
  }
  kc = std::min(kc, Hkv);
  CopyStreams cs;
  rc = copy_streams(&cs);
  if (rc != SSKIP_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t row = (size_t)L * d * 2;  // bytes of one head's [L, d] bf16 matrix
  const int n_groups = (Hkv + kc - 1) / kc;
  const int n_chunks = B * n_groups;
  // ev[2c]: chunk c copied in; ev[2c + 1]: chunk c computed; then start, the
  // end of the copies out and the end of the copies in.
  std::vector<cudaEvent_t> ev(2 * n_chunks + 3, nullptr);
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      rc = SSKIP_ERR_CUDA;
      break;
    }
  if (rc == SSKIP_OK && skip_count &&
      cudaMemsetAsync(skip_count, 0, 2 * sizeof(unsigned long long), st) != cudaSuccess)
    rc = SSKIP_ERR_CUDA;
  // Copies start only after the work already queued on the caller's stream.
  if (rc == SSKIP_OK && (cudaEventRecord(ev[2 * n_chunks], st) != cudaSuccess ||
                         cudaStreamWaitEvent(cs.in, ev[2 * n_chunks], 0) != cudaSuccess ||
                         cudaStreamWaitEvent(cs.out, ev[2 * n_chunks], 0) != cudaSuccess))
    rc = SSKIP_ERR_CUDA;
  auto h2d = [&](void* dst, const void* src, size_t off, size_t n) {
    return cudaMemcpyAsync(static_cast<char*>(dst) + off, static_cast<const char*>(src) + off, n,
                           cudaMemcpyHostToDevice, cs.in) == cudaSuccess;
  };
  auto d2h = [&](void* dst, const void* src, size_t off, size_t n) {
    return cudaMemcpyAsync(static_cast<char*>(dst) + off, static_cast<const char*>(src) + off, n,
                           cudaMemcpyDeviceToHost, cs.out) == cudaSuccess;
  };
  for (int c = 0; rc == SSKIP_OK && c < n_chunks; ++c) {
    const int b = c / n_groups, kv0 = (c % n_groups) * kc, nk = std::min(kc, Hkv - kv0);
    const size_t qo = ((size_t)b * Hq + (size_t)kv0 * G) * row, qn = (size_t)nk * G * row;
    const size_t ko = ((size_t)b * Hkv + kv0) * row, kn = (size_t)nk * row;
    const size_t lo = ((size_t)b * Hq + (size_t)kv0 * G) * L * 4, ln = (size_t)nk * G * L * 4;
    if (!h2d(q_d, q_h, qo, qn) || !h2d(k_d, k_h, ko, kn) || !h2d(v_d, v_h, ko, kn) ||
        cudaEventRecord(ev[2 * c], cs.in) != cudaSuccess ||
        cudaStreamWaitEvent(st, ev[2 * c], 0) != cudaSuccess) {
      rc = SSKIP_ERR_CUDA;
      break;
    }
    rc = prefill_impl(static_cast<const char*>(q_d) + qo, static_cast<const char*>(k_d) + ko,
                      static_cast<const char*>(v_d) + ko, static_cast<char*>(o_d) + qo,
                      reinterpret_cast<float*>(reinterpret_cast<char*>(lse_d) + lo), 1, nk * G, nk,
                      L, d, causal, sm_scale, threshold_scale_factor, Br, Bc, Br, skip_count, 2,
                      nullptr, nullptr, nullptr, stream, /*zero_counts=*/false);
    if (rc != SSKIP_OK) break;
    if (cudaEventRecord(ev[2 * c + 1], st) != cudaSuccess ||
        cudaStreamWaitEvent(cs.out, ev[2 * c + 1], 0) != cudaSuccess ||
        !d2h(o_h, o_d, qo, qn) ||
        !d2h(lse_h, lse_d, lo, ln))
      rc = SSKIP_ERR_CUDA;
  }
  // The caller's stream completes only after every copy this call enqueued,
  // on an error path as well: a caller that frees or reuses the buffers after
  // an error must not race with copies still in flight.
  if (ev[2 * n_chunks + 2]) {
    const bool joined = cudaEventRecord(ev[2 * n_chunks + 1], cs.out) == cudaSuccess &&
                        cudaStreamWaitEvent(st, ev[2 * n_chunks + 1], 0) == cudaSuccess &&
                        cudaEventRecord(ev[2 * n_chunks + 2], cs.in) == cudaSuccess &&
                        cudaStreamWaitEvent(st, ev[2 * n_chunks + 2], 0) == cudaSuccess;
    if (!joined && rc == SSKIP_OK) rc = SSKIP_ERR_CUDA;
  }
  for (auto& e : ev)
    if (e) cudaEventDestroy(e);  // released once the recorded work completes
  return rc;
}

SSKIP_API int sskip_attn_decode_host(const void* q_h, const int* seqlens_h, void* o_h, float* lse_h,
                                     void* q_d, int* seqlens_d, void* o_d, float* lse_d,
                                     const void* kcache, const void* vcache, int B, int Hq,
                                     int Hkv, int Lmax, int d, float sm_scale,
                                     float threshold_scale_factor, int Bc, int num_splits,
                                     void* workspace, size_t workspace_bytes,
                                     unsigned long long* skip_count, void* stream) {
  if (!q_h || !seqlens_h || !o_h || !lse_h || !q_d || !seqlens_d || !o_d || !lse_d)
    return SSKIP_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || (d != 64 && d != 128)) return SSKIP_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t qn = (size_t)B * Hq * d * 2, ln = (size_t)B * Hq * 4;
  if (cudaMemcpyAsync(q_d, q_h, qn, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(seqlens_d, seqlens_h, (size_t)B * 4, cudaMemcpyHostToDevice, st) !=
          cudaSuccess)
    return SSKIP_ERR_CUDA;
  const int rc = sskip_attn_decode_ex(q_d, kcache, vcache, seqlens_d, o_d, lse_d, B, Hq, Hkv,
                                      Lmax, d, sm_scale, threshold_scale_factor, Bc, num_splits,
                                      workspace, workspace_bytes, skip_count, nullptr, stream);
  if (rc != SSKIP_OK) return rc;
  if (cudaMemcpyAsync(o_h, o_d, qn, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(lse_h, lse_d, ln, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return SSKIP_ERR_CUDA;
  return SSKIP_OK;
}
