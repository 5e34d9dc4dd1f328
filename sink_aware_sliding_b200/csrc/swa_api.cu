// C ABI of libswa: argument checks, TMA descriptors, launch configuration.
// Declarations and contracts: include/swa.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/swa.h"
#include "based_linear.h"
#include "swa_internal.h"

namespace {

// Device error word: kernels set it (first writer wins) when a bounded wait expires.
__device__ int g_swa_error;

std::atomic<unsigned long long> g_timeout_ns{2000000000ull};
std::atomic<int> g_debug_flags{0};

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int decode_ctas_per_sm[2] = {0, 0};  // d = 64, 128 (for B <= 4096 table)
  int* err = nullptr;
};
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiled g_encode = nullptr;

int device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SWA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SWA_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_swa_error) != cudaSuccess) return SWA_ERR_CUDA;
    d.err = static_cast<int*>(p);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return SWA_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiled>(fn);
    }
    d.ready = true;
  }
  *out = &d;
  return SWA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 3-D tiled map over a [rows, heads, d] tensor: box = {128 bytes of d, 1 head, box_rows}.
// atom32: 128-byte swizzle with 32-byte atoms (fp32 operands read in MN-major order).
int make_map(CUtensorMap* m, const void* ptr, bool f32, int d, int heads, long long rows,
             int box_rows, bool atom32 = false) {
  const int elem = f32 ? 4 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * elem,
                           static_cast<cuuint64_t>(d) * elem * heads};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem), 1u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                        const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        atom32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SWA_OK : SWA_ERR_CUDA;
}

int check_heads(int Hq, int Hkv, int d, int window, int n_sink, float scale, int dtype) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return SWA_ERR_INVALID_ARG;
  if (window < 1 || n_sink < 0) return SWA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return SWA_ERR_INVALID_ARG;
  if (dtype != SWA_DTYPE_BF16 && dtype != SWA_DTYPE_F32 && dtype != SWA_DTYPE_BF16_F32OUT)
    return SWA_ERR_INVALID_ARG;
  if (d <= 0) return SWA_ERR_INVALID_ARG;
  if (dtype != SWA_DTYPE_F32 && d != 64 && d != 128) return SWA_ERR_UNSUPPORTED;
  if (dtype == SWA_DTYPE_F32 && d != 64) return SWA_ERR_UNSUPPORTED;
  return SWA_OK;
}

int run_prefill(const void* q, const void* k, const void* v, void* out, float* lse,
                const int32_t* cu, int n_seq, int L, long long T, int Hq, int Hkv, int d,
                int window, int n_sink, float scale, int dtype, cudaStream_t stream) {
  DeviceInfo* dev = nullptr;
  int st = device_info(&dev);
  if (st != SWA_OK) return st;
  const bool f32 = dtype == SWA_DTYPE_F32;
  CUtensorMap tq, tk, tv, to;
  std::memset(&to, 0, sizeof(to));
  if ((st = make_map(&tq, q, f32, d, Hq, T, swa::kBM)) != SWA_OK) return st;
  if (dtype == SWA_DTYPE_BF16 && (st = make_map(&to, out, false, d, Hq, T, swa::kBM)) != SWA_OK) return st;
  if ((st = make_map(&tk, k, f32, d, Hkv, T, swa::kBN)) != SWA_OK) return st;
  if ((st = make_map(&tv, v, f32, d, Hkv, T, swa::kBN, f32)) != SWA_OK) return st;
  swa::PrefillArgs a{};
  a.out = out;
  a.lse = lse;
  a.cu_seqlens = cu;
  a.n_seq = n_seq;
  a.L = L;
  a.T = T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.window = window;
  a.n_sink = n_sink;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.lse_varlen = cu != nullptr ? 1 : 0;
  a.timeout_ns = g_timeout_ns.load();
  a.debug_flags = g_debug_flags.load();
  a.err = dev->err;
  long long units;
  if (cu == nullptr) {
    const long long tiles = static_cast<long long>(n_seq) * ((L + swa::kBM - 1) / swa::kBM);
    if (tiles * Hq > INT32_MAX) return SWA_ERR_UNSUPPORTED;
    a.total_tiles = static_cast<int>(tiles);
    units = tiles * Hq;
  } else {
    a.total_tiles = -1;
    units = (T / swa::kBM + n_seq) * static_cast<long long>(Hq);  // upper bound
    if (units > INT32_MAX) return SWA_ERR_UNSUPPORTED;
  }
  // Debug flag 4 skips the short-window stream kernel, flag 2 forces the one-tile
  // kernel (so tests can check every kernel on the same inputs).
  if ((a.debug_flags & 6) == 0 && swa::prefill_stream_supported(d, f32, window, n_sink)) {
    const int grid_s = static_cast<int>(std::min<long long>(dev->sms, units));
    cudaError_t es = swa::launch_prefill_stream(a, tq, tk, tv, to, dtype != SWA_DTYPE_BF16, grid_s, stream);
    if (es != cudaErrorNotSupported) return es == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
  }
  const bool pair = (a.debug_flags & 2) == 0 && swa::prefill_pair_supported(Hq, Hq / Hkv, d, f32);
  if (pair) units = (units + 1) / 2;
  const int grid = static_cast<int>(std::min<long long>(dev->sms, units));
  if (grid <= 0) return SWA_OK;
  cudaError_t e = cudaErrorNotSupported;
  if (pair) e = swa::launch_prefill_pair(a, tq, tk, tv, to, d, f32, dtype != SWA_DTYPE_BF16, grid, stream);
  if (e == cudaErrorNotSupported) {  // one-tile kernel (odd Hq, or the two-tile kernel declined)
    const int grid1 = static_cast<int>(std::min<long long>(dev->sms, pair ? 2 * units : units));
    e = swa::launch_prefill(a, tq, tk, tv, d, f32, dtype != SWA_DTYPE_BF16, grid1, stream);
  }
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

// Split-K decode grid: one warp per kDecodeKeysPerWarp keys of the largest
// possible visible set (every segment holds at most window + n_sink keys; the
// positions themselves are on the device), and never more CTAs than fill the GPU.
constexpr long long kDecodeKeysPerWarp = 64;
int decode_grid(DeviceInfo* dev, int d, int B, int Hkv, int window, int n_sink, int* grid) {
  const int idx = d == 128 ? 1 : 0;
  if (dev->decode_ctas_per_sm[idx] == 0) {
    int c = 0;
    if (swa::decode_occupancy(d, 4096, &c) != cudaSuccess || c <= 0) return SWA_ERR_CUDA;
    dev->decode_ctas_per_sm[idx] = c;
  }
  const long long full = static_cast<long long>(dev->sms) * dev->decode_ctas_per_sm[idx];
  const long long max_keys = static_cast<long long>(B) * Hkv * (static_cast<long long>(window) + n_sink);
  const long long warps = (max_keys + kDecodeKeysPerWarp - 1) / kDecodeKeysPerWarp;
  const long long wpc = swa::decode_threads() / 32;
  *grid = static_cast<int>(std::max(1LL, std::min(full, (warps + wpc - 1) / wpc)));
  return SWA_OK;
}

}  // namespace

extern "C" {

int swa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
            int Hkv, int L, int d, int window, int n_sink, float scale, int dtype,
            swa_stream_t stream) {
  int st = check_heads(Hq, Hkv, d, window, n_sink, scale, dtype);
  if (st != SWA_OK) return st;
  if (B < 0 || L < 0) return SWA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * L == 0) return SWA_OK;
  if (!q || !k || !v || !out) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return SWA_ERR_INVALID_ARG;
  const long long T = static_cast<long long>(B) * L;
  if (T > INT32_MAX) return SWA_ERR_UNSUPPORTED;
  return run_prefill(q, k, v, out, lse, nullptr, B, L, T, Hq, Hkv, d, window, n_sink, scale, dtype,
                     reinterpret_cast<cudaStream_t>(stream));
}

int swa_fwd_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                   const int32_t* cu_seqlens, int n_seq, long long T, int Hq, int Hkv, int d,
                   int window, int n_sink, float scale, int dtype, swa_stream_t stream) {
  int st = check_heads(Hq, Hkv, d, window, n_sink, scale, dtype);
  if (st != SWA_OK) return st;
  if (n_seq < 1 || T < 0 || !cu_seqlens) return SWA_ERR_INVALID_ARG;
  if (n_seq > swa::kMaxSeqSmem) return SWA_ERR_UNSUPPORTED;
  if (T > INT32_MAX) return SWA_ERR_UNSUPPORTED;
  if (T == 0) return SWA_OK;
  if (!q || !k || !v || !out) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return SWA_ERR_INVALID_ARG;
  return run_prefill(q, k, v, out, lse, cu_seqlens, n_seq, 0, T, Hq, Hkv, d, window, n_sink, scale,
                     dtype, reinterpret_cast<cudaStream_t>(stream));
}

static int check_cache(int B, int Hkv, int d, int window, int n_sink, const void* kc,
                       const void* vc, const void* sk, const void* sv) {
  if (B < 0 || Hkv <= 0 || window < 1 || n_sink < 0) return SWA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SWA_ERR_UNSUPPORTED;
  if (!kc || !vc || !aligned16(kc) || !aligned16(vc)) return SWA_ERR_INVALID_ARG;
  if (n_sink > 0 && (!sk || !sv || !aligned16(sk) || !aligned16(sv))) return SWA_ERR_INVALID_ARG;
  return SWA_OK;
}

int swa_cache_fill(const void* k, const void* v, int P, void* kcache, void* vcache, void* sink_k,
                   void* sink_v, int B, int Hkv, int d, int window, int n_sink,
                   swa_stream_t stream) {
  int st = check_cache(B, Hkv, d, window, n_sink, kcache, vcache, sink_k, sink_v);
  if (st != SWA_OK) return st;
  if (P < 0) return SWA_ERR_INVALID_ARG;
  if (P == 0 || B == 0) return SWA_OK;
  if (!k || !v || !aligned16(k) || !aligned16(v)) return SWA_ERR_INVALID_ARG;
  cudaError_t e = swa::launch_cache_fill(k, v, P, kcache, vcache, sink_k, sink_v, B, Hkv, d, window,
                                         n_sink, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

int swa_cache_append(const void* k_new, const void* v_new, const int32_t* pos, void* kcache,
                     void* vcache, void* sink_k, void* sink_v, int B, int Hkv, int d, int window,
                     int n_sink, swa_stream_t stream) {
  int st = check_cache(B, Hkv, d, window, n_sink, kcache, vcache, sink_k, sink_v);
  if (st != SWA_OK) return st;
  if (B == 0) return SWA_OK;
  if (!k_new || !v_new || !pos || !aligned16(k_new) || !aligned16(v_new) ||
      (reinterpret_cast<uintptr_t>(pos) & 3u))
    return SWA_ERR_INVALID_ARG;
  cudaError_t e = swa::launch_cache_append(k_new, v_new, pos, kcache, vcache, sink_k, sink_v, B, Hkv,
                                           d, window, n_sink, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

static int decode_shape_ok(int B, int Hq, int Hkv, int d, int window, int n_sink) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || window < 1 || n_sink < 0)
    return SWA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SWA_ERR_UNSUPPORTED;
  if (Hq / Hkv > 8) return SWA_ERR_UNSUPPORTED;
  if (B > 4096) return SWA_ERR_UNSUPPORTED;
  return SWA_OK;
}

size_t swa_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int window, int n_sink) {
  if (decode_shape_ok(B, Hq, Hkv, d, window, n_sink) != SWA_OK) return 0;
  DeviceInfo* dev = nullptr;
  if (device_info(&dev) != SWA_OK) return 0;
  int grid = 0;
  if (decode_grid(dev, d, B, Hkv, window, n_sink, &grid) != SWA_OK) return 0;
  const size_t n_warps = static_cast<size_t>(grid) * (swa::decode_threads() / 32);
  const size_t slots = n_warps + static_cast<size_t>(B) * Hkv;
  return slots * swa::decode_partial_floats(Hq / Hkv, d) * sizeof(float);
}

}  // extern "C"

namespace swa {

int decode_args_status(const void* q, const void* kcache, const void* vcache, const void* sink_k,
                       const void* sink_v, const int32_t* pos, const void* out, const float* lse, int B,
                       int Hq, int Hkv, int d, int window, int n_sink, float scale, int out_dtype) {
  int st = decode_shape_ok(B, Hq, Hkv, d, window, n_sink);
  if (st != SWA_OK) return st;
  if (!(scale > 0.f) || !std::isfinite(scale)) return SWA_ERR_INVALID_ARG;
  if (out_dtype != SWA_DTYPE_BF16 && out_dtype != SWA_DTYPE_BF16_F32OUT) return SWA_ERR_INVALID_ARG;
  if (B == 0) return SWA_OK;
  if (!q || !pos || !out || !aligned16(q) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(pos) & 3u) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return SWA_ERR_INVALID_ARG;
  return check_cache(B, Hkv, d, window, n_sink, kcache, vcache, sink_k, sink_v);
}

}  // namespace swa

extern "C" {

static int run_decode(const void* q, const void* kcache, const void* vcache, const void* sink_k,
                      const void* sink_v, const int32_t* pos, void* out, float* lse, int B, int Hq,
                      int Hkv, int d, int window, int n_sink, float scale, int out_dtype, void* workspace,
                      size_t workspace_bytes, const swa::RopeTable* rope, swa_stream_t stream) {
  int st = swa::decode_args_status(q, kcache, vcache, sink_k, sink_v, pos, out, lse, B, Hq, Hkv, d, window,
                                   n_sink, scale, out_dtype);
  if (st != SWA_OK) return st;
  if (B == 0) return SWA_OK;
  const size_t need = swa_decode_workspace_bytes(B, Hq, Hkv, d, window, n_sink);
  if (need == 0) return SWA_ERR_CUDA;
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SWA_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != SWA_OK) return st;
  int grid = 0;
  if ((st = decode_grid(dev, d, B, Hkv, window, n_sink, &grid)) != SWA_OK) return st;
  swa::DecodeArgs a{};
  a.q = q;
  a.kcache = kcache;
  a.vcache = vcache;
  a.sink_k = sink_k;
  a.sink_v = sink_v;
  a.pos = pos;
  a.out = out;
  a.lse = lse;
  a.part = static_cast<float*>(workspace);
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.W = window;
  a.S = n_sink;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.n_warps = grid * (swa::decode_threads() / 32);
  a.out_f32 = out_dtype == SWA_DTYPE_BF16_F32OUT ? 1 : 0;
  cudaError_t e = swa::launch_decode(a, d, grid, swa::decode_threads(),
                                     reinterpret_cast<cudaStream_t>(stream), rope);
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

int swa_decode(const void* q, const void* kcache, const void* vcache, const void* sink_k,
               const void* sink_v, const int32_t* pos, void* out, float* lse, int B, int Hq,
               int Hkv, int d, int window, int n_sink, float scale, void* workspace,
               size_t workspace_bytes, swa_stream_t stream) {
  return run_decode(q, kcache, vcache, sink_k, sink_v, pos, out, lse, B, Hq, Hkv, d, window, n_sink,
                    scale, SWA_DTYPE_BF16, workspace, workspace_bytes, nullptr, stream);
}

int swa_decode_ex(const void* q, const void* kcache, const void* vcache, const void* sink_k,
                  const void* sink_v, const int32_t* pos, void* out, float* lse, int B, int Hq, int Hkv,
                  int d, int window, int n_sink, float scale, int out_dtype, void* workspace,
                  size_t workspace_bytes, swa_stream_t stream) {
  return run_decode(q, kcache, vcache, sink_k, sink_v, pos, out, lse, B, Hq, Hkv, d, window, n_sink,
                    scale, out_dtype, workspace, workspace_bytes, nullptr, stream);
}

static bool rope_base_ok(double base) { return base > 0.0 && std::isfinite(base); }

int swa_decode_rope(const void* q, const void* kcache, const void* vcache, const void* sink_k,
                    const void* sink_v, const int32_t* pos, void* out, float* lse, int B, int Hq,
                    int Hkv, int d, int window, int n_sink, float scale, double rope_base,
                    void* workspace, size_t workspace_bytes, swa_stream_t stream) {
  if (!rope_base_ok(rope_base)) return SWA_ERR_INVALID_ARG;
  swa::RopeTable rt;
  swa::make_rope_table(rope_base, d, &rt);
  return run_decode(q, kcache, vcache, sink_k, sink_v, pos, out, lse, B, Hq, Hkv, d, window, n_sink,
                    scale, SWA_DTYPE_BF16, workspace, workspace_bytes, &rt, stream);
}

int swa_rope_qk(void* q, void* k, const int32_t* positions, long long n_tokens, int Hq, int Hkv, int d,
                double rope_base, swa_stream_t stream) {
  if (n_tokens < 0 || Hq < 0 || (k != nullptr && Hkv < 0) || !rope_base_ok(rope_base))
    return SWA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SWA_ERR_UNSUPPORTED;
  if (n_tokens == 0 || (Hq == 0 && (k == nullptr || Hkv == 0))) return SWA_OK;
  if (!positions || (reinterpret_cast<uintptr_t>(positions) & 3u) || (Hq > 0 && (!q || !aligned16(q))) ||
      (k != nullptr && !aligned16(k)))
    return SWA_ERR_INVALID_ARG;
  swa::RopeTable rt;
  swa::make_rope_table(rope_base, d, &rt);
  cudaError_t e = swa::launch_rope_qk(Hq > 0 ? q : nullptr, k, positions, n_tokens, Hq, k ? Hkv : 0, d, rt,
                                      reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

int swa_rope_cache_append(const void* k_new, const void* v_new, const int32_t* pos, void* kcache,
                          void* vcache, void* sink_k, void* sink_v, int B, int Hkv, int d, int window,
                          int n_sink, double rope_base, swa_stream_t stream) {
  if (!rope_base_ok(rope_base)) return SWA_ERR_INVALID_ARG;
  int st = check_cache(B, Hkv, d, window, n_sink, kcache, vcache, sink_k, sink_v);
  if (st != SWA_OK) return st;
  if (B == 0) return SWA_OK;
  if (!k_new || !v_new || !pos || !aligned16(k_new) || !aligned16(v_new) ||
      (reinterpret_cast<uintptr_t>(pos) & 3u))
    return SWA_ERR_INVALID_ARG;
  swa::RopeTable rt;
  swa::make_rope_table(rope_base, d, &rt);
  cudaError_t e = swa::launch_rope_append(k_new, v_new, pos, kcache, vcache, sink_k, sink_v, B, Hkv, d,
                                          window, n_sink, rt, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

int swa_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
            float* dq, float* dk, float* dv, int B, int Hq, int Hkv, int L, int d, int window, int n_sink,
            float scale, swa_stream_t stream) {
  int st = check_heads(Hq, Hkv, d, window, n_sink, scale, SWA_DTYPE_BF16);
  if (st != SWA_OK) return st;
  if (B < 0 || L < 0) return SWA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * L == 0) return SWA_OK;
  const void* ptrs[9] = {q, k, v, out, dout, dq, dk, dv, nullptr};
  for (int i = 0; i < 8; ++i)
    if (!ptrs[i] || !aligned16(ptrs[i])) return SWA_ERR_INVALID_ARG;
  if (!lse || (reinterpret_cast<uintptr_t>(lse) & 3u)) return SWA_ERR_INVALID_ARG;
  const long long T = static_cast<long long>(B) * L;
  if (T > INT32_MAX || T * Hq > INT32_MAX) return SWA_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != SWA_OK) return st;
  CUtensorMap tq, tk, tv, tdo;
  if ((st = make_map(&tq, q, false, d, Hq, T, swa::kBM)) != SWA_OK) return st;
  if ((st = make_map(&tk, k, false, d, Hkv, T, swa::kBN)) != SWA_OK) return st;
  if ((st = make_map(&tv, v, false, d, Hkv, T, swa::kBN)) != SWA_OK) return st;
  if ((st = make_map(&tdo, dout, false, d, Hq, T, swa::kBM)) != SWA_OK) return st;
  swa::BwdArgs ba{};
  swa::PrefillArgs& a = ba.pa;
  a.n_seq = B;
  a.L = L;
  a.T = T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.window = window;
  a.n_sink = n_sink;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.total_tiles = static_cast<int>(static_cast<long long>(B) * ((L + swa::kBM - 1) / swa::kBM));
  a.timeout_ns = g_timeout_ns.load();
  a.debug_flags = g_debug_flags.load();
  a.err = dev->err;
  ba.out = out;
  ba.dout = dout;
  ba.lse = lse;
  ba.dq = dq;
  ba.dk = dk;
  ba.dv = dv;
  cudaError_t e = swa::launch_bwd(ba, tq, tk, tv, tdo, d, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

int swa_hybrid_decode(const void* q, const void* k_new, const void* v_new, const int32_t* pos, void* kcache,
                      void* vcache, void* sink_k, void* sink_v, void* out, float* lse, int B, int Hq, int Hkv,
                      int d, int window, int n_sink, float scale, const void* ql, const void* kl, const void* vl,
                      float* state, float* zsum, void* out_l, int H_l, int dk, int dv, float scale_l,
                      swa_stream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || window < 1 || n_sink < 0 || H_l <= 0)
    return SWA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale) || !(scale_l > 0.f) || !std::isfinite(scale_l))
    return SWA_ERR_INVALID_ARG;
  if (!swa::hybrid_window_supported(d, window, n_sink) || dk != 16 || dv != 64) return SWA_ERR_UNSUPPORTED;
  if (B == 0) return SWA_OK;
  const void* ptrs[] = {q, k_new, v_new, kcache, vcache, out, ql, kl, vl, state, zsum, out_l};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return SWA_ERR_INVALID_ARG;
  if (n_sink > 0 && (!sink_k || !sink_v || !aligned16(sink_k) || !aligned16(sink_v))) return SWA_ERR_INVALID_ARG;
  if (!pos || (reinterpret_cast<uintptr_t>(pos) & 3u) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return SWA_ERR_INVALID_ARG;
  swa::HybridArgs a{};
  a.q = q;
  a.k_new = k_new;
  a.v_new = v_new;
  a.pos = pos;
  a.kcache = kcache;
  a.vcache = vcache;
  a.sink_k = sink_k;
  a.sink_v = sink_v;
  a.out = out;
  a.lse = lse;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.W = window;
  a.S = n_sink;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.ql = ql;
  a.kl = kl;
  a.vl = vl;
  a.state = state;
  a.zsum = zsum;
  a.out_l = out_l;
  a.H_l = H_l;
  a.scale_l = scale_l;
  cudaError_t e = swa::launch_hybrid_decode(a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

int swa_based_linear_state_features(int dk) { return dk > 0 ? swa::based_linear_features(dk) : 0; }

int swa_based_linear_fwd(const void* q, const void* k, const void* v, void* out, float* state, float* zsum,
                         int B, int L, int H, int dk, int dv, float scale, int out_dtype, swa_stream_t stream) {
  if (B < 0 || L < 0 || H <= 0 || !(scale > 0.f) || !std::isfinite(scale)) return SWA_ERR_INVALID_ARG;
  if (out_dtype != SWA_DTYPE_BF16 && out_dtype != SWA_DTYPE_F32) return SWA_ERR_INVALID_ARG;
  if (dk != 16 || dv != 64) return SWA_ERR_UNSUPPORTED;
  if ((state == nullptr) != (zsum == nullptr)) return SWA_ERR_INVALID_ARG;
  // L = 0 still writes the (zero) state when one is asked for
  if (B == 0 || (L == 0 && state == nullptr)) return SWA_OK;
  if (L > 0 && (!q || !k || !v || !out || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)))
    return SWA_ERR_INVALID_ARG;
  if (state != nullptr && !aligned16(state)) return SWA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > INT32_MAX) return SWA_ERR_UNSUPPORTED;
  DeviceInfo* di = nullptr;
  const int st = device_info(&di);
  if (st != SWA_OK) return st;
  swa::BasedLinearArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.state = state;
  a.zsum = zsum;
  a.B = B;
  a.L = L;
  a.H = H;
  a.scale = scale;
  a.out_f32 = out_dtype == SWA_DTYPE_F32 ? 1 : 0;
  a.timeout_ns = g_timeout_ns.load();
  a.debug_flags = g_debug_flags.load();
  a.err = di->err;
  cudaError_t e = swa::launch_based_linear_fwd(a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

int swa_based_linear_decode(const void* q, const void* k, const void* v, float* state, float* zsum, void* out,
                            int B, int H, int dk, int dv, float scale, int out_dtype, swa_stream_t stream) {
  if (B < 0 || H <= 0 || !(scale > 0.f) || !std::isfinite(scale)) return SWA_ERR_INVALID_ARG;
  if (out_dtype != SWA_DTYPE_BF16 && out_dtype != SWA_DTYPE_F32) return SWA_ERR_INVALID_ARG;
  if (dk != 16 || dv != 64) return SWA_ERR_UNSUPPORTED;
  if (B == 0) return SWA_OK;
  if (!q || !k || !v || !state || !zsum || !out || !aligned16(state)) return SWA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > INT32_MAX) return SWA_ERR_UNSUPPORTED;
  cudaError_t e = swa::launch_based_linear_decode(q, k, v, state, zsum, out, B, H, scale, out_dtype == SWA_DTYPE_F32,
                                                  reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

int swa_hadamard_proj(const void* y, const float* alpha, const float* beta, void* z,
                      long long n_rows, int n, int out_dtype, swa_stream_t stream) {
  if (n_rows < 0 || n < 32 || n > 8192 || (n & (n - 1)) != 0) return n_rows < 0 ? SWA_ERR_INVALID_ARG
                                                                      : SWA_ERR_UNSUPPORTED;
  if (out_dtype != SWA_DTYPE_BF16 && out_dtype != SWA_DTYPE_F32) return SWA_ERR_INVALID_ARG;
  if (n_rows == 0) return SWA_OK;
  if (!y || !alpha || !beta || !z || !aligned16(y) || !aligned16(alpha) || !aligned16(beta) ||
      !aligned16(z))
    return SWA_ERR_INVALID_ARG;
  DeviceInfo* di = nullptr;
  const int st = device_info(&di);
  if (st != SWA_OK) return st;
  swa::HadamardArgs a;
  a.y = y;
  a.alpha = alpha;
  a.beta = beta;
  a.z = z;
  a.n_rows = n_rows;
  a.timeout_ns = g_timeout_ns.load();
  a.debug_flags = g_debug_flags.load();
  a.err = di->err;
  cudaError_t e = swa::launch_hadamard(a, n, out_dtype == SWA_DTYPE_F32, di->sms,
                                       reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

const char* swa_status_string(int status) {
  switch (status) {
    case SWA_OK: return "ok";
    case SWA_ERR_INVALID_ARG: return "invalid argument";
    case SWA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SWA_ERR_CUDA: return "CUDA error";
    case SWA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case SWA_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int swa_device_error(swa_stream_t stream) {
  DeviceInfo* dev = nullptr;
  int st = device_info(&dev);
  if (st != SWA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SWA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, dev->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SWA_ERR_CUDA;
  const int zero = 0;
  if (v != 0 && cudaMemcpy(dev->err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return SWA_ERR_CUDA;
  return v;
}

int swa_debug_error_word(swa_stream_t stream) { return swa_device_error(stream); }

unsigned long long swa_set_wait_timeout_ns(unsigned long long ns) { return g_timeout_ns.exchange(ns); }

int swa_set_debug_flags(int flags) { return g_debug_flags.exchange(flags); }

int swa_version(void) { return 0x000100; }

}  // extern "C"
