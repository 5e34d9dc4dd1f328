// Pieces shared by the prefill kernels: work-unit decoding (which key tiles a
// query tile visits), bounded barrier waits, the per-tile online softmax on a
// row held in tensor memory, and the epilogue that writes O and LSE.
//
// Visible set ("Sliding-window beats linear attention", sections 1 and 3):
// row t sees key j iff j <= t and (j >= t - window + 1 or j < n_sink).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"
#include "swa_internal.h"

namespace swa {
namespace prefill {

constexpr int kStatusTimeout = 4;  // SWA_ERR_DEVICE_TIMEOUT

// One query tile of one head: rows [m0, m1] of sequence seq, and its key tiles:
// first the nst tiles of the sink prefix that lie left of the band, then the
// band tiles kb_lo .. kb_lo + n_tiles - nst - 1.
struct Unit {
  int seq, seq_start, len, m0, m1, nst, kb_lo, n_tiles;
};

struct Ctl {
  volatile int* abort_flag;
  const PrefillArgs* a;
};

__device__ __forceinline__ void fail(const Ctl& c) {
  *c.abort_flag = 1;
  atomicCAS(c.a->err, 0, kStatusTimeout);
}

// Bounded wait on (bar, parity).  False if the time limit ran out (which starts
// the CTA's abort) or, when honor_abort is set, as soon as another thread has
// started it.  Teardown waits pass honor_abort = false.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, Ctl c, bool honor_abort = true) {
  for (int i = 0; i < 256; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (honor_abort && *c.abort_flag) return false;
    if (globaltimer_ns() - t0 > c.a->timeout_ns) {
      fail(c);
      return false;
    }
  }
}

// Query tile number gt (0 = first tile of the first sequence) -> unit geometry.
// Varlen sequences are found in the shared tables: s_cu (cu_seqlens copy) and
// s_tpre (query tiles before each sequence).
__device__ __forceinline__ void decode_tile(const PrefillArgs& a, const int* s_cu, const int* s_tpre,
                                            int gt, Unit& x) {
  int qt;
  if (a.cu_seqlens == nullptr) {
    const int tps = (a.L + kBM - 1) / kBM;
    x.seq = gt / tps;
    qt = gt - x.seq * tps;
    x.seq_start = x.seq * a.L;
    x.len = a.L;
  } else {
    int lo = 0, hi = a.n_seq - 1;  // last sequence with s_tpre[seq] <= gt (skips empty ones)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_tpre[mid] <= gt) lo = mid; else hi = mid - 1;
    }
    x.seq = lo;
    qt = gt - s_tpre[lo];
    x.seq_start = s_cu[lo];
    x.len = s_cu[lo + 1] - s_cu[lo];
  }
  x.m0 = qt * kBM;
  x.m1 = min(x.m0 + kBM, x.len) - 1;
  const int lo_key = max(0, x.m0 - a.window + 1);
  x.kb_lo = lo_key / kBN;
  const int kb_hi = x.m1 / kBN;
  x.nst = a.n_sink > 0 ? min((a.n_sink + kBN - 1) / kBN, x.kb_lo) : 0;
  x.n_tiles = x.nst + kb_hi - x.kb_lo + 1;
}

__device__ __forceinline__ int tile_n0(const Unit& x, int j) {
  return (j < x.nst ? j : x.kb_lo + (j - x.nst)) * kBN;
}

// Does key tile j of unit x hold any key some row of the tile cannot see?
__device__ __forceinline__ bool tile_needs_mask(const Unit& x, int j, int window) {
  const int n0 = tile_n0(x, j);
  return (j < x.nst) || (n0 + kBN - 1 > x.m0) || (n0 < x.m1 - window + 1);
}

// Warp 0 builds the varlen tables (cu_seqlens copy and query-tile prefix sums).
__device__ __forceinline__ void build_varlen_tables(const PrefillArgs& a, int* s_cu, int* s_tpre,
                                                    int lane) {
  const int n = a.n_seq;
  const int per = (n + 31) / 32;
  int local = 0;
  for (int i = lane * per; i < min(n, (lane + 1) * per); ++i) {
    const int c0 = a.cu_seqlens[i], c1 = a.cu_seqlens[i + 1];
    s_cu[i] = c0;
    local += (c1 - c0 + kBM - 1) / kBM;
  }
  if (lane == 0) s_cu[n] = a.cu_seqlens[n];
  int incl = local;
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  int run = incl - local;
  for (int i = lane * per; i < min(n, (lane + 1) * per); ++i) {
    s_tpre[i] = run;
    run += (a.cu_seqlens[i + 1] - a.cu_seqlens[i] + kBM - 1) / kBM;
  }
  if (lane == 31) s_tpre[n] = incl;
}

// Online softmax of one key tile for the row this thread owns (TMEM lane).
// Reads S from s_tmem (128 fp32 columns), masks it if the tile needs it,
// moves the reference max only when it grew by more than 2^8 in exp2 units,
// writes P over S (packed bf16 pairs, or fp32 for the tf32 path) and updates
// the running max and sum.  Returns whether the reference max moved; alpha is
// the factor the row's O accumulator must be scaled by in that case.
// Bits [a, b] (inclusive, clipped to the word) of the 32-column word starting at column base.
__device__ __forceinline__ uint32_t range_bits(int a, int b, int base) {
  const int lo = max(a - base, 0), hi = min(b - base, 31);
  if (lo > hi) return 0u;
  return (0xFFFFFFFFu >> (31 - hi)) & (0xFFFFFFFFu << lo);
}

// Set the columns of s this row cannot see to -inf.  Visible: c <= hi and
// (c >= lo or c < sk), all relative to the tile's first key.  The visible columns
// are first gathered into four 32-bit words (two ranges per word), then every
// column is kept or cleared by its bit: one code path of two instructions per
// column for every kind of edge tile (diagonal, lower band edge, sink prefix).
__device__ __forceinline__ void mask_tile(float* s, int hi, int lo, int sk) {
  uint32_t w[kBN / 32];
#pragma unroll
  for (int k = 0; k < kBN / 32; ++k)
    w[k] = range_bits(max(lo, 0), hi, 32 * k) | range_bits(0, min(sk, hi + 1) - 1, 32 * k);
#pragma unroll
  for (int c = 0; c < kBN; ++c)
    s[c] = (static_cast<int>(w[c >> 5] << (31 - (c & 31))) < 0) ? s[c] : -INFINITY;
}

// Online softmax of one key tile for the row this thread owns (TMEM lane).
// Reads S from s_tmem (128 fp32 columns), masks it if the tile needs it,
// moves the reference max only when it grew by more than 2^8 in exp2 units,
// writes P over S (packed bf16 pairs, or fp32 for the tf32 path) and updates
// the running max and sum.  Returns whether the reference max moved; alpha is
// the factor the row's O accumulator must be scaled by in that case.
template <bool F32>
__device__ __forceinline__ bool softmax_tile(uint32_t s_tmem, const Unit& x, int j, int t,
                                             const PrefillArgs& a, float& m_run, float& l_run,
                                             float& alpha) {
  const float sl2 = a.scale_log2;
  float s[kBN];
  {
    uint32_t sr[kBN];
    tmem_ld128_wait(s_tmem, sr);
#pragma unroll
    for (int i = 0; i < kBN; ++i) s[i] = __uint_as_float(sr[i]);
  }
  if (tile_needs_mask(x, j, a.window)) {
    const int n0 = tile_n0(x, j);
    mask_tile(s, t - n0, t - a.window + 1 - n0, a.n_sink - n0);
  }
  // row max: 8 chains of three-input max
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = fmaxf(s[2 * i], s[2 * i + 1]);
#pragma unroll
  for (int c = 16; c < kBN; c += 16)
#pragma unroll
    for (int i = 0; i < 8; ++i) mx[i] = max3(mx[i], s[c + 2 * i], s[c + 2 * i + 1]);
  const float m_tile = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
  const float m_new = fmaxf(m_run, m_tile);
  // NaN from (-inf) - (-inf) compares false: a row with nothing visible yet keeps -inf.
  const bool need = (m_new - m_run) * sl2 > 8.0f;
  const float m_use = need ? m_new : m_run;
  alpha = need ? ex2_approx((m_run - m_new) * sl2) : 1.0f;
  const float neg = (m_use == -INFINITY) ? 0.0f : -m_use * sl2;
  // p = 2^(s * scale * log2 e - m * scale * log2 e): the argument on pairs, exp2 on the MUFU
  const uint64_t scale2 = f2_pack(sl2, sl2), neg2 = f2_pack(neg, neg);
  uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
  for (int i = 0; i < kBN / 2; ++i) {
    float x0, x1;
    f2_unpack(f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), scale2, neg2), x0, x1);
    s[2 * i] = ex2_approx(x0);
    s[2 * i + 1] = ex2_approx(x1);
    acc[i & 3] = f2_add(acc[i & 3], f2_pack(s[2 * i], s[2 * i + 1]));
  }
  float sum0, sum1, sum2, sum3;
  f2_unpack(f2_add(acc[0], acc[1]), sum0, sum1);
  f2_unpack(f2_add(acc[2], acc[3]), sum2, sum3);
  l_run = l_run * alpha + ((sum0 + sum1) + (sum2 + sum3));
  m_run = m_use;
  if constexpr (F32) {
#pragma unroll
    for (int c = 0; c < kBN / 32; ++c) {
      uint32_t pr[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) pr[i] = __float_as_uint(s[c * 32 + i]);
      tmem_st32(s_tmem + c * 32, pr);
    }
  } else {
#pragma unroll
    for (int c = 0; c < kBN / 64; ++c) {
      uint32_t pr[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) pr[i] = pack_bf16x2(s[c * 64 + 2 * i], s[c * 64 + 2 * i + 1]);
      tmem_st32(s_tmem + c * 32, pr);
    }
  }
  return need;
}

// Sink mini-tile.  A sink prefix of at most kSinkMini keys whose key tile lies
// left of the band (the band starts at key 128 or later) is not run as a masked
// 128-key tile: Q K^T is formed on the first 16 keys only (N = 16), the softmax
// works on 16 columns, and P V is one K = 16 product.  Every row sees every sink
// then (rows are past key 127), so the mask is just c < n_sink.  The K and V tiles
// are still loaded whole; only their first 16 rows are read.
constexpr int kSinkMini = 16;
__device__ __forceinline__ bool sink_mini(const Unit& x, int n_sink) {
  return x.nst == 1 && n_sink <= kSinkMini;
}

// Online softmax of the sink mini-tile (bf16 path): S columns 0..15 at s_tmem, P
// (8 packed bf16 pairs) written over columns 0..7.  Same running max, sum and
// rescale rule as softmax_tile.
__device__ __forceinline__ bool softmax_sink16(uint32_t s_tmem, int n_sink, float sl2, float& m_run,
                                               float& l_run, float& alpha) {
  float s[kSinkMini];
  {
    uint32_t sr[kSinkMini];
    tmem_ld16_wait(s_tmem, sr);
#pragma unroll
    for (int c = 0; c < kSinkMini; ++c) s[c] = c < n_sink ? __uint_as_float(sr[c]) : -INFINITY;
  }
  float mx[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) mx[i] = max3(s[i], s[4 + i], fmaxf(s[8 + i], s[12 + i]));
  const float m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
  const float m_new = fmaxf(m_run, m_tile);
  const bool need = (m_new - m_run) * sl2 > 8.0f;
  const float m_use = need ? m_new : m_run;
  alpha = need ? ex2_approx((m_run - m_new) * sl2) : 1.0f;
  const float neg = (m_use == -INFINITY) ? 0.0f : -m_use * sl2;
  const uint64_t scale2 = f2_pack(sl2, sl2), neg2 = f2_pack(neg, neg);
  uint64_t acc[2] = {0, 0};
  uint32_t pr[kSinkMini / 2];
#pragma unroll
  for (int i = 0; i < kSinkMini / 2; ++i) {
    float x0, x1;
    f2_unpack(f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), scale2, neg2), x0, x1);
    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
    acc[i & 1] = f2_add(acc[i & 1], f2_pack(p0, p1));
    pr[i] = pack_bf16x2(p0, p1);
  }
  float sum0, sum1, sum2, sum3;
  f2_unpack(acc[0], sum0, sum1);
  f2_unpack(acc[1], sum2, sum3);
  l_run = l_run * alpha + ((sum0 + sum1) + (sum2 + sum3));
  m_run = m_use;
  tmem_st8(s_tmem, pr);
  return need;
}

// Scale this warp's 32 rows of O (d columns at o_tmem) by alpha (per row).
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t o_tmem, float alpha) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t rr[32];
    tmem_ld32_wait(o_tmem + c * 32, rr);
    const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float lo, hi;
      f2_unpack(f2_mul(f2_pack(__uint_as_float(rr[2 * i]), __uint_as_float(rr[2 * i + 1])), a2), lo, hi);
      rr[2 * i] = __float_as_uint(lo);
      rr[2 * i + 1] = __float_as_uint(hi);
    }
    tmem_st32(o_tmem + c * 32, rr);
  }
}

// O / l of this thread's row (d columns at o_tmem) -> out, and the row's LSE.
template <int D, bool OUT_F32>
__device__ __forceinline__ void store_row(uint32_t o_tmem, const PrefillArgs& a, const Unit& x,
                                          int h, int t, float m_run, float l_run) {
  const bool valid = t < x.len;
  const float inv_l = 1.0f / l_run;
  const size_t row = static_cast<size_t>(x.seq_start) + static_cast<size_t>(t);
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t rr[32];
    tmem_ld32_wait(o_tmem + c * 32, rr);
    if (!valid) continue;
    if constexpr (OUT_F32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + (row * a.Hq + h) * D + c * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        dst[i] = make_float4(__uint_as_float(rr[4 * i]) * inv_l, __uint_as_float(rr[4 * i + 1]) * inv_l,
                             __uint_as_float(rr[4 * i + 2]) * inv_l, __uint_as_float(rr[4 * i + 3]) * inv_l);
    } else {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + (row * a.Hq + h) * D + c * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(rr[8 * i + 0]) * inv_l, __uint_as_float(rr[8 * i + 1]) * inv_l);
        w.y = pack_bf16x2(__uint_as_float(rr[8 * i + 2]) * inv_l, __uint_as_float(rr[8 * i + 3]) * inv_l);
        w.z = pack_bf16x2(__uint_as_float(rr[8 * i + 4]) * inv_l, __uint_as_float(rr[8 * i + 5]) * inv_l);
        w.w = pack_bf16x2(__uint_as_float(rr[8 * i + 6]) * inv_l, __uint_as_float(rr[8 * i + 7]) * inv_l);
        dst[i] = w;
      }
    }
  }
  if (valid && a.lse != nullptr) {
    const float ref = (m_run == -INFINITY) ? 0.0f : m_run * a.scale_log2;
    const float lse = (ref + log2f(l_run)) * 0.69314718055994531f;
    const size_t idx = a.lse_varlen ? static_cast<size_t>(h) * static_cast<size_t>(a.T) + row
                                    : (static_cast<size_t>(x.seq) * a.Hq + h) * a.L + t;
    a.lse[idx] = lse;
  }
}

// O / l of this thread's row, as bf16, into a 128-row x 128-byte shared tile in
// the 128-byte swizzled layout the output tensor map stores from (d = 64), and
// the row's LSE to global memory.
__device__ __forceinline__ void stage_row_bf16_d64(uint32_t o_tmem, uint8_t* tile, int r,
                                                   const PrefillArgs& a, const Unit& x, int h, int t,
                                                   float m_run, float l_run) {
  const float inv_l = 1.0f / l_run;
  const uint64_t s2 = f2_pack(inv_l, inv_l);
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    uint32_t rr[32];
    tmem_ld32_wait(o_tmem + c * 32, rr);
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // 16-byte chunk 4c+q of the row: columns 32c+8q .. +7
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float lo, hi;
        f2_unpack(f2_mul(f2_pack(__uint_as_float(rr[8 * q + 2 * e]), __uint_as_float(rr[8 * q + 2 * e + 1])), s2),
                  lo, hi);
        w[e] = pack_bf16x2(lo, hi);
      }
      const int chunk = 4 * c + q;
      *reinterpret_cast<uint4*>(tile + r * 128 + ((chunk ^ (r & 7)) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  if (t < x.len && a.lse != nullptr) {
    const size_t row = static_cast<size_t>(x.seq_start) + static_cast<size_t>(t);
    const float ref = (m_run == -INFINITY) ? 0.0f : m_run * a.scale_log2;
    const float lse = (ref + log2f(l_run)) * 0.69314718055994531f;
    const size_t idx = a.lse_varlen ? static_cast<size_t>(h) * static_cast<size_t>(a.T) + row
                                    : (static_cast<size_t>(x.seq) * a.Hq + h) * a.L + t;
    a.lse[idx] = lse;
  }
}

// Descriptor arithmetic for the MMA issue loops.  The start-address field of a
// shared-memory descriptor holds (address >> 4) in its low 14 bits, and every
// shared address here lies below 2^18, so adding (bytes >> 4) to a descriptor moves
// its start by `bytes` without touching the other fields.  The issue loops build
// one descriptor per tile and step through it with compile-time offsets (in a
// one-CTA microbenchmark on a B200, tcgen05.mma instructions whose descriptors
// needed run-time address arithmetic issued at about 90 cycles each, against the
// tensor pipe's 52 with base + constant).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }
// Offset of K-major k-step kk (32 bytes) in a tile of `rows` rows stored as 128-byte
// column chunks (STEPS_PER_CHUNK k-steps per chunk).
template <int STEPS_PER_CHUNK, int ROWS>
__host__ __device__ constexpr uint32_t kmajor_off(int kk) {
  return static_cast<uint32_t>((kk / STEPS_PER_CHUNK) * (ROWS * 128) + (kk % STEPS_PER_CHUNK) * 32);
}
// Offset of MN-major k-step kk of KSTEP rows (128 bytes per row).
template <int KSTEP>
__host__ __device__ constexpr uint32_t mnmajor_off(int kk) {
  return static_cast<uint32_t>(kk * KSTEP * 128);
}

// Shared-memory matrix descriptors of the operands (see the kernels for the layouts).
// K-major tile of `rows` rows x (NCHUNK x 128 bytes), 128-byte swizzle: MMA k-step kk of
// 32 bytes lies in column chunk kk / steps_per_chunk.
template <int STEPS_PER_CHUNK>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_base, int rows, int kk) {
  const int ch = kk / STEPS_PER_CHUNK;
  const int wi = kk % STEPS_PER_CHUNK;
  return smem_desc(tile_base + ch * (rows * 128) + wi * 32, 16, 1024, kLayoutSw128);
}
// V as the MN-major B operand of O += P V: k-step kk covers KSTEP key rows; LBO jumps
// between 128-byte column chunks of d (kBN rows apart); SBO between swizzle atoms along
// the keys (8 rows; tf32 operands in MN-major order need the 32-byte-atom swizzle whose
// atom is 4 rows).
template <bool F32, int KSTEP>
__device__ __forceinline__ uint64_t v_desc(uint32_t tile_base, int kk) {
  return F32 ? smem_desc(tile_base + kk * (KSTEP * 128), kBN * 128, 512, kLayoutSw128Atom32)
             : smem_desc(tile_base + kk * (KSTEP * 128), kBN * 128, 1024, kLayoutSw128);
}

}  // namespace prefill
}  // namespace swa
