// Decode step over the ring-buffer KV cache, split over the GPU's warps.
//
// For one new token per sequence (query q [B, Hq, d] at position pos[b]) the
// visible keys are the ring slots holding positions max(0, pos-W+1)..pos and
// the sink slots j < min(S, pos-W+1) ("Sliding-window beats linear
// attention", sections 1 and 3).  Per (b, kvh) that is a segment of
//     len_b = min(pos_b + 1, W) + clamp(pos_b - W + 1, 0, S)
// keys, shared by the G = Hq/Hkv query heads of the KV head.
//
// Split-K without load imbalance: the segments of all (b, kvh) are laid end to
// end and the concatenated key range is cut into equal contiguous pieces, one
// per warp of a grid that fills every SM.  A warp walks its piece in blocks of
// 16 keys, keeps an online softmax per head, and writes one partial state
// (unnormalised O, running max, running sum) whenever it leaves a segment.
// swa_decode_merge_kernel then combines the partials of each segment by their
// log-sum-exps.
//
// The inner loop is bound by HBM: every cache row is read once with 128-bit
// non-caching loads straight into registers.  The two small products per
// block (S = Q K^T with the G heads padded to 16 rows, and O^T += V^T P^T) run
// as mma.sync m16n8k16 bf16 instructions only to keep the instruction issue
// far below the load rate; the dims are permuted consistently between q, k and
// the output so that every fragment comes from whole 16-byte loads.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "ptx.cuh"
#include "rope.cuh"
#include "swa_internal.h"

namespace swa {
namespace {

constexpr int kDecodeThreads = 128;

struct SegTable {
  const long long* pre;  // pre[b] = sum_{b' < b} len_b'  (B + 1 entries)
};

__device__ __forceinline__ int seg_len(int p, int W, int S) {
  const int ring = min(p + 1, W);
  const int sinks = min(max(p - W + 1, 0), S);
  return ring + sinks;
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}
// Pack bf16 element e of a with bf16 element e of b (a in the low half).
__device__ __forceinline__ uint32_t pair(const uint4& a, const uint4& b, int e) {
  return __byte_perm(word(a, e >> 1), word(b, e >> 1), (e & 1) ? 0x7632 : 0x5410);
}

// Number of pieces the K concatenated keys are cut into: one per warp of the grid,
// but no more than one per kMinPieceKeys keys, so that no piece is empty (each piece
// has at least one key whenever pieces <= K) and short contexts are not spread thin.
constexpr long long kMinPieceKeys = 16;
__device__ __forceinline__ long long effective_pieces(long long K, long long n_warps) {
  return max(1LL, min(n_warps, (K + kMinPieceKeys - 1) / kMinPieceKeys));
}

// Binary search: the batch b whose segments [pre[b]*Hkv, pre[b+1]*Hkv) hold key x.
__device__ __forceinline__ int find_batch(const long long* pre, int B, long long x, int Hkv) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] * Hkv <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int D>
struct DCfg {
  static constexpr int KCH = D / 32;  // 16-byte K chunks per thread and key row
  static constexpr int KS = D / 16;   // k-steps of S = Q K^T
  static constexpr int VCH = D / 64;  // 16-byte V chunks per thread and key row (1 or 2)
  static constexpr int MT = D / 16;   // m-tiles of O^T
};

template <int D>
struct Block {
  uint4 k[2][DCfg<D>::KCH];   // keys g and g+8 of the block, dims chunked as described above
  uint4 v[4][DCfg<D>::VCH];   // keys 2t, 2t+1, 2t+8, 2t+9
};

template <int D, bool ROPE>
__global__ void __launch_bounds__(kDecodeThreads)
    swa_decode_split_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ RopeTable rt) {
  using C = DCfg<D>;
  extern __shared__ long long s_pre[];  // B + 1
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int B = a.B, W = a.W, S = a.S, Hkv = a.Hkv, G = a.G;

  // Per-batch segment-length prefix (warp 0), shared by the CTA.
  if (threadIdx.x < 32) {
    const int per = (B + 31) / 32;
    long long local = 0;
    for (int b = lane * per; b < min(B, (lane + 1) * per); ++b) local += seg_len(a.pos[b], W, S);
    long long incl = local;
    for (int off = 1; off < 32; off <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    long long run = incl - local;
    for (int b = lane * per; b < min(B, (lane + 1) * per); ++b) {
      s_pre[b] = run;
      run += seg_len(a.pos[b], W, S);
    }
    if (lane == 31) s_pre[B] = incl;
  }
  __syncthreads();

  const long long K = s_pre[B] * Hkv;
  const long long Wn = effective_pieces(K, a.n_warps);
  const long long wid = static_cast<long long>(blockIdx.x) * (kDecodeThreads / 32) + (threadIdx.x >> 5);
  if (wid >= Wn) return;                 // fewer keys than the grid was sized for: idle warp
  long long x = wid * K / Wn;
  const long long x_end = (wid + 1) * K / Wn;
  const size_t part_floats = static_cast<size_t>(G) * (D + 2);
  const float sl2 = a.scale_log2;

  while (x < x_end) {
    const int b = find_batch(s_pre, B, x, Hkv);
    const int p = a.pos[b];
    const long long len = s_pre[b + 1] - s_pre[b];
    const int kvh = static_cast<int>((x - s_pre[b] * Hkv) / len);
    const long long off = s_pre[b] * Hkv + kvh * len;
    const int k0 = static_cast<int>(x - off);
    const int k1 = static_cast<int>(min(x_end, off + len) - off);
    const int nring = min(p + 1, W);
    const size_t seg = static_cast<size_t>(b) * Hkv + kvh;
    const __nv_bfloat16* kr = static_cast<const __nv_bfloat16*>(a.kcache) + seg * W * D;
    const __nv_bfloat16* vr = static_cast<const __nv_bfloat16*>(a.vcache) + seg * W * D;
    const __nv_bfloat16* ks = static_cast<const __nv_bfloat16*>(a.sink_k) + seg * S * D;
    const __nv_bfloat16* vs = static_cast<const __nv_bfloat16*>(a.sink_v) + seg * S * D;
    auto krow = [&](int i) { return i < nring ? kr + static_cast<size_t>(i) * D : ks + static_cast<size_t>(i - nring) * D; };
    auto vrow = [&](int i) { return i < nring ? vr + static_cast<size_t>(i) * D : vs + static_cast<size_t>(i - nring) * D; };

    // Q fragments (A of S = Q K^T): row g = head g of this KV head, same dim chunks as K.
    uint32_t qa[C::KS][2];
    {
      const bool real = g < G;
      const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(a.q) +
                                  (static_cast<size_t>(b) * a.Hq + kvh * G + (real ? g : 0)) * D;
      uint4 w[C::KCH];
#pragma unroll
      for (int c = 0; c < C::KCH; ++c)
        w[c] = real ? *reinterpret_cast<const uint4*>(qrow + c * 32 + t * 8) : make_uint4(0, 0, 0, 0);
      if constexpr (ROPE) {
        // rotate-half partner of element c*32 + t*8 + e is in chunk c + KCH/2 of the same thread
        if (real)
#pragma unroll
          for (int c = 0; c < C::KCH / 2; ++c) rope_rotate_chunks(w[c], w[c + C::KCH / 2], p, c * 32 + t * 8, rt.theta);
      }
#pragma unroll
      for (int c = 0; c < C::KCH; ++c) {
        qa[2 * c][0] = w[c].x; qa[2 * c][1] = w[c].y;
        qa[2 * c + 1][0] = w[c].z; qa[2 * c + 1][1] = w[c].w;
      }
    }
    float o[C::MT][4];
#pragma unroll
    for (int i = 0; i < C::MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;   // head g, in log2 units of scaled scores

    auto load = [&](Block<D>& blk, int kb) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = kb + h * 8 + g;
#pragma unroll
        for (int c = 0; c < C::KCH; ++c)
          blk.k[h][c] = i < k1 ? ldg_stream(krow(i) + c * 32 + t * 8) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = kb + 2 * t + (r & 1) + (r >> 1) * 8;
#pragma unroll
        for (int c = 0; c < C::VCH; ++c)
          blk.v[r][c] = i < k1 ? ldg_stream(vrow(i) + c * 64 + g * 8) : make_uint4(0, 0, 0, 0);
      }
    };

    auto compute = [&](const Block<D>& blk, int kb) {
      float sc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int s = 0; s < C::KS; ++s) {
          const uint4& kw = blk.k[nt][s >> 1];
          const uint32_t b0 = (s & 1) ? kw.z : kw.x;
          const uint32_t b1 = (s & 1) ? kw.w : kw.y;
          mma_bf16(sc[nt], qa[s][0], 0u, qa[s][1], 0u, b0, b1);
        }
      }
      // scores of head g for keys kb + {2t, 2t+1, 8+2t, 9+2t}, in log2 units
      float z[4] = {sc[0][0] * sl2, sc[0][1] * sl2, sc[1][0] * sl2, sc[1][1] * sl2};
      const int kidx[4] = {kb + 2 * t, kb + 2 * t + 1, kb + 8 + 2 * t, kb + 9 + 2 * t};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (kidx[i] >= k1) z[i] = -INFINITY;
      float mx = fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run, mx);
      const float alpha = (m_new == -INFINITY) ? 1.f : ex2_approx(m_run - m_new);
      const float ref = (m_new == -INFINITY) ? 0.f : m_new;
      float pz[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) pz[i] = ex2_approx(z[i] - ref);
      l_run = l_run * alpha + ((pz[0] + pz[1]) + (pz[2] + pz[3]));
      m_run = m_new;
      const bool real = g < G;
      const uint32_t pb0 = real ? pack_bf16x2(pz[0], pz[1]) : 0u;
      const uint32_t pb1 = real ? pack_bf16x2(pz[2], pz[3]) : 0u;
      const float a_lo = __shfl_sync(0xffffffffu, alpha, (2 * t) * 4);
      const float a_hi = __shfl_sync(0xffffffffu, alpha, (2 * t + 1) * 4);
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) {
        o[mt][0] *= a_lo; o[mt][1] *= a_hi; o[mt][2] *= a_lo; o[mt][3] *= a_hi;
        uint32_t va0, va1, va2, va3;
        if constexpr (D == 128) {
          va0 = pair(blk.v[0][0], blk.v[1][0], mt);
          va1 = pair(blk.v[0][1], blk.v[1][1], mt);
          va2 = pair(blk.v[2][0], blk.v[3][0], mt);
          va3 = pair(blk.v[2][1], blk.v[3][1], mt);
        } else {
          va0 = pair(blk.v[0][0], blk.v[1][0], mt);
          va1 = pair(blk.v[0][0], blk.v[1][0], 4 + mt);
          va2 = pair(blk.v[2][0], blk.v[3][0], mt);
          va3 = pair(blk.v[2][0], blk.v[3][0], 4 + mt);
        }
        mma_bf16(o[mt], va0, va1, va2, va3, pb0, pb1);
      }
    };

    Block<D> b0, b1;
    int kb = k0;
    load(b0, kb);
    while (true) {
      const bool more1 = kb + 16 < k1;
      if (more1) load(b1, kb + 16);
      compute(b0, kb);
      kb += 16;
      if (!more1) break;
      const bool more0 = kb + 16 < k1;
      if (more0) load(b0, kb + 16);
      compute(b1, kb);
      kb += 16;
      if (!more0) break;
    }

    // Partial state of this (segment, warp): slot wid + seg.
    float* part = a.part + (static_cast<size_t>(wid) + seg) * part_floats;
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    if (t == 0 && g < G) {
      part[G * D + g] = m_run;
      part[G * D + G + g] = l_run;
    }
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) {
      const int dA = (D == 128) ? g * 8 + mt : g * 8 + mt;
      const int dB = (D == 128) ? 64 + g * 8 + mt : g * 8 + 4 + mt;
      const int h0 = 2 * t, h1 = 2 * t + 1;
      if (h0 < G) {
        part[h0 * D + dA] = o[mt][0];
        part[h0 * D + dB] = o[mt][2];
      }
      if (h1 < G) {
        part[h1 * D + dA] = o[mt][1];
        part[h1 * D + dB] = o[mt][3];
      }
    }
    x = off + k1;
  }
}

// One CTA per (b, kvh) segment and query head h of that KV head: combine the partials
// of the pieces that covered the segment by their log-sum-exps.  Pieces w_first ..
// w_last of the concatenated key range overlap the segment (none is empty, see
// effective_pieces).  kMergeSplit x D threads: thread (s, dim) sums output element dim
// over the pieces p = s mod kMergeSplit, eight loads in flight, so that a segment
// cut into many pieces (a single long sequence) is not a long chain of dependent
// loads; the kMergeSplit partial sums are then added in shared memory.  With few
// pieces per segment (many sequences) kMergeSplit = 1 keeps the CTAs small.
template <int D, int kMergeSplit>
__global__ void __launch_bounds__(kMergeSplit * D) swa_decode_merge_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int kThreads = kMergeSplit * D;
  const int seg = blockIdx.x;
  const int h = blockIdx.y;
  const int b = seg / a.Hkv, kvh = seg % a.Hkv;
  const int G = a.G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int dim = tid % D, split = tid / D;
  __shared__ long long s_red[kThreads / 32][2];
  __shared__ float s_wmax[kThreads / 32];
  __shared__ float s_e[kThreads];
  __shared__ float s_el[kThreads];
  __shared__ float s_acc[kMergeSplit][D];
  __shared__ float s_l[kMergeSplit][D];
  // Offset of this segment in the concatenated key range, and the total.
  long long before = 0, total = 0;
  for (int i = tid; i < a.B; i += kThreads) {
    const long long l = seg_len(a.pos[i], a.W, a.S);
    total += l;
    if (i < b) before += l;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, o);
    total += __shfl_xor_sync(0xffffffffu, total, o);
  }
  if (lane == 0) {
    s_red[warp][0] = before;
    s_red[warp][1] = total;
  }
  __syncthreads();
  before = total = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) {
    before += s_red[w][0];
    total += s_red[w][1];
  }
  const long long len = seg_len(a.pos[b], a.W, a.S);
  const long long off = before * a.Hkv + kvh * len;
  const long long K = total * a.Hkv;
  const long long Wn = effective_pieces(K, a.n_warps);
  const long long w_first = ((off + 1) * Wn - 1) / K;   // piece holding key off
  const long long w_last = ((off + len) * Wn - 1) / K;  // piece holding key off + len - 1
  const int np = static_cast<int>(w_last - w_first + 1);
  const size_t part_floats = static_cast<size_t>(G) * (D + 2);
  const float* part0 = a.part + (static_cast<size_t>(w_first) + seg) * part_floats;

  // 1. this head's reference max over the pieces
  float m = -INFINITY;
  for (int p = tid; p < np; p += kThreads) m = fmaxf(m, part0[p * part_floats + G * D + h]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) s_wmax[warp] = m;
  __syncthreads();
  float M = s_wmax[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) M = fmaxf(M, s_wmax[w]);

  // 2. weighted sums, kThreads pieces' weights staged at a time
  float acc = 0.f, lacc = 0.f;
  for (int c0 = 0; c0 < np; c0 += kThreads) {
    {
      const int p = c0 + tid;
      float e = 0.f, el = 0.f;
      if (p < np) {
        const float* pp = part0 + p * part_floats;
        e = ex2_approx(pp[G * D + h] - M);
        el = e * pp[G * D + G + h];
      }
      s_e[tid] = e;
      s_el[tid] = el;
    }
    __syncthreads();
    const int n = min(kThreads, np - c0);
    const float* pp = part0 + static_cast<size_t>(c0) * part_floats + h * D + dim;
    for (int p0 = split; p0 < n; p0 += 8 * kMergeSplit) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int p = p0 + u * kMergeSplit;
        v[u] = p < n ? pp[p * part_floats] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int p = p0 + u * kMergeSplit;
        if (p < n) {
          acc += s_e[p] * v[u];
          lacc += s_el[p];
        }
      }
    }
    __syncthreads();
  }
  s_acc[split][dim] = acc;
  s_l[split][dim] = lacc;
  __syncthreads();
  if (split == 0) {
#pragma unroll
    for (int s2 = 1; s2 < kMergeSplit; ++s2) {
      acc += s_acc[s2][dim];
      lacc += s_l[s2][dim];
    }
    const size_t orow = static_cast<size_t>(b) * a.Hq + kvh * G + h;
    const float o = acc / lacc;
    if (a.out_f32)
      static_cast<float*>(a.out)[orow * D + dim] = o;
    else
      static_cast<__nv_bfloat16*>(a.out)[orow * D + dim] = __float2bfloat16_rn(o);
    if (dim == 0 && a.lse != nullptr) a.lse[orow] = (M + log2f(lacc)) * 0.69314718055994531f;
  }
}

template <int D>
cudaError_t launch_decode_impl(const DecodeArgs& a, int grid, int block, cudaStream_t stream,
                               const RopeTable* rope) {
  const size_t smem = sizeof(long long) * (a.B + 1);
  if (rope != nullptr) {
    swa_decode_split_kernel<D, true><<<grid, block, smem, stream>>>(a, *rope);
  } else {
    const RopeTable unused{};
    swa_decode_split_kernel<D, false><<<grid, block, smem, stream>>>(a, unused);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // pieces per segment when the sequences are equally long: the grid's warps over the segments
  const long long pieces = a.n_warps / (static_cast<long long>(a.B) * a.Hkv) + 1;
  if (pieces > 16)
    swa_decode_merge_kernel<D, 4><<<dim3(a.B * a.Hkv, a.G), 4 * D, 0, stream>>>(a);
  else
    swa_decode_merge_kernel<D, 1><<<dim3(a.B * a.Hkv, a.G), D, 0, stream>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- ring cache
// One thread per 16 bytes of a (b, position, head) row.
__global__ void swa_cache_fill_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                      int P, uint4* kc, uint4* vc, uint4* sk, uint4* sv, int B,
                                      int Hkv, int vec, int W, int S) {
  const int n_ring = min(P, W);
  const int n_sink = min(P, S);
  const long long rows = static_cast<long long>(B) * (n_ring + n_sink) * Hkv;
  const long long total = rows * vec;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int e = static_cast<int>(i % vec);
    long long r = i / vec;
    const int h = static_cast<int>(r % Hkv);
    r /= Hkv;
    const int pi = static_cast<int>(r % (n_ring + n_sink));
    const int b = static_cast<int>(r / (n_ring + n_sink));
    const bool ring = pi < n_ring;
    const int p = ring ? P - n_ring + pi : pi - n_ring;
    const size_t src = ((static_cast<size_t>(b) * P + p) * Hkv + h) * vec + e;
    const size_t seg = static_cast<size_t>(b) * Hkv + h;
    if (ring) {
      const size_t dst = (seg * W + (p % W)) * vec + e;
      kc[dst] = k[src];
      vc[dst] = v[src];
    } else {
      const size_t dst = (seg * S + p) * vec + e;
      sk[dst] = k[src];
      sv[dst] = v[src];
    }
  }
}

__global__ void swa_cache_append_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                        const int32_t* __restrict__ pos, uint4* kc, uint4* vc,
                                        uint4* sk, uint4* sv, int B, int Hkv, int vec, int W,
                                        int S) {
  const long long total = static_cast<long long>(B) * Hkv * vec;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int e = static_cast<int>(i % vec);
    const long long bh = i / vec;
    const int b = static_cast<int>(bh / Hkv);
    const int p = pos[b];
    if (p < 0) continue;
    const uint4 kx = k[i], vx = v[i];
    const size_t dst = (static_cast<size_t>(bh) * W + (p % W)) * vec + e;
    kc[dst] = kx;
    vc[dst] = vx;
    if (p < S) {
      const size_t ds = (static_cast<size_t>(bh) * S + p) * vec + e;
      sk[ds] = kx;
      sv[ds] = vx;
    }
  }
}

}  // namespace

size_t decode_partial_floats(int G, int d) { return static_cast<size_t>(G) * (d + 2); }

cudaError_t launch_decode(const DecodeArgs& a, int d, int grid, int block, cudaStream_t stream,
                          const RopeTable* rope) {
  if (d == 128) return launch_decode_impl<128>(a, grid, block, stream, rope);
  if (d == 64) return launch_decode_impl<64>(a, grid, block, stream, rope);
  return cudaErrorInvalidValue;
}

cudaError_t decode_occupancy(int d, int B, int* ctas_per_sm) {
  const size_t smem = sizeof(long long) * (B + 1);
  if (d == 128)
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, swa_decode_split_kernel<128, false>,
                                                         kDecodeThreads, smem);
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, swa_decode_split_kernel<64, false>,
                                                       kDecodeThreads, smem);
}

int decode_threads() { return kDecodeThreads; }

cudaError_t launch_cache_fill(const void* k, const void* v, int P, void* kc, void* vc, void* sk,
                              void* sv, int B, int Hkv, int d, int W, int S, cudaStream_t stream) {
  const int vec = d / 8;
  const long long total = static_cast<long long>(B) * (min(P, W) + min(P, S)) * Hkv * vec;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const long long blocks = std::min<long long>((total + threads - 1) / threads, 148LL * 64);
  swa_cache_fill_kernel<<<static_cast<int>(blocks), threads, 0, stream>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), P, static_cast<uint4*>(kc),
      static_cast<uint4*>(vc), static_cast<uint4*>(sk), static_cast<uint4*>(sv), B, Hkv, vec, W, S);
  return cudaGetLastError();
}

cudaError_t launch_cache_append(const void* k, const void* v, const int32_t* pos, void* kc,
                                void* vc, void* sk, void* sv, int B, int Hkv, int d, int W, int S,
                                cudaStream_t stream) {
  const int vec = d / 8;
  const long long total = static_cast<long long>(B) * Hkv * vec;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const long long blocks = std::min<long long>((total + threads - 1) / threads, 148LL * 16);
  swa_cache_append_kernel<<<static_cast<int>(blocks), threads, 0, stream>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), pos, static_cast<uint4*>(kc),
      static_cast<uint4*>(vc), static_cast<uint4*>(sk), static_cast<uint4*>(sv), B, Hkv, vec, W, S);
  return cudaGetLastError();
}

}  // namespace swa
