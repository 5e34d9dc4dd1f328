// Backward pass of sink-aware sliding-window attention, sm_100a (d = 64 or 128,
// bf16 inputs, fp32 gradients).  The visible set is the forward's ("Sliding-window
// beats linear attention", sections 1 and 3): row t sees key j iff j <= t and
// (j >= t - window + 1 or j < n_sink).  With P the forward's softmax (recomputed
// from the saved log-sum-exp) and D_t = rowsum(dO_t * O_t):
//     dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.
//
// Two kernels, neither needing atomics:
//   swa_bwd_dkdv_kernel  one CTA per (sequence, KV head, 128-key tile): for every
//                        query head of that KV head and every query tile that sees
//                        the key tile (the band, or all later tiles for a tile
//                        holding sinks) it computes S^T = K Q^T and dP^T = V dO^T on
//                        tcgen05, forms P^T and dS^T per key row (thread = TMEM lane =
//                        key), and accumulates dV += P^T dO and dK += dS^T Q in TMEM;
//   swa_bwd_dq_kernel    one CTA per (sequence, query head, 128-row query tile): for
//                        the key tiles the forward visits it computes S and dP, forms
//                        dS per query row and accumulates dQ += dS K in TMEM.
// A third, small kernel computes D_t = rowsum(dO_t O_t) for every row first,
// into the storage of dq (which the dQ kernel only writes after the dK/dV kernel
// has read D; the dQ kernel forms its own D per row).
// Each CTA has two element-wise warpgroups over the same 128 TMEM lanes: the first
// does the element-wise step on score columns 0-63, the second on columns 64-127
// (the step is independent per column), so each thread handles half a row.
// Visibility is tested only on edge tiles, through four 32-bit words per row built
// from the row's visible column ranges (a separate code path for fully visible
// tiles).  Every hand-off is an mbarrier with a bounded wait.  In both kernels a
// ninth warp issues TMA and MMA, so the element-wise warps wait only for their
// scores.  In the dK/dV kernel the accumulation products of one iteration and the
// score products of the next go out back to back, Q and dO are double-buffered and
// requested two iterations ahead, and the products and the element-wise step of one
// iteration run one after another (TMEM holds one iteration's scores next to the
// two accumulators).  In the dQ kernel dS has TMEM columns of its own, so the score
// products of the next key tile run during the element-wise step; K is kept in
// three buffers and V in two.
//
// TMEM (dK/dV kernel): S^T 0-127, dP^T 128-255 (P^T and dS^T, packed bf16, are
// written over columns 0-31 and 64-95 of each, every warpgroup within the columns
// it read), dV 256.., dK 256+d..; (dQ kernel): S 0-127, dP 128-255, dQ 256..,
// dS packed at 384-415 and 448-479.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "prefill_common.cuh"

namespace swa {
namespace {

using namespace prefill;

constexpr int kEwThreads = 256;    // the element-wise threads of both kernels (warps 0-7)

template <int D>
struct BwdCfg {
  static constexpr int TILE = kBM * D * 2;             // one 128-row bf16 tile
  static constexpr int NCHUNK = D / 64;                // 128-byte column chunks
  static constexpr int QK_STEPS = D / 16;
  static constexpr int PV_STEPS = kBN / 16;
  // shared layout: tiles 0..5 (two fixed, two double-buffered), then the dK/dV
  // kernel's row data (two slots of 128 D + 128 lse floats), then barriers
  static constexpr int OFF_T = 0;
  static constexpr int OFF_STG = 6 * TILE;
  static constexpr int OFF_BAR = OFF_STG + 2048;
  static constexpr int NBAR = 9;
  static constexpr int OFF_TMEMPTR = OFF_BAR + 8 * NBAR;
  // Each CTA allocates all 512 TMEM columns, so no second CTA may share the SM
  // (its allocation would have to wait): ask for more than half of the SM's
  // shared memory even where the tiles need less.
  static constexpr int SMEM_USED = OFF_TMEMPTR + 16 + 1024;
  static constexpr int SMEM_BYTES = SMEM_USED > 119808 ? SMEM_USED : 119808;
  static constexpr uint32_t IDESC_SS = make_idesc(1u, kBM, kBN, false);   // 128 x 128 scores
  static constexpr uint32_t IDESC_ACC = make_idesc(1u, kBM, D, true);     // 128 x d accumulators
};

// dQ kernel layout: Q, dO, three K buffers, two V buffers (K is read by both the score
// and the accumulation products, so it is kept one key tile longer), then barriers.
template <int D>
struct DqCfg : BwdCfg<D> {
  using B = BwdCfg<D>;
  static constexpr int OFF_K = 2 * B::TILE;
  static constexpr int OFF_V = 5 * B::TILE;
  static constexpr int OFF_BAR = 7 * B::TILE;
  static constexpr int NBAR = 11;
  static constexpr int OFF_TMEMPTR = OFF_BAR + 8 * NBAR;
  static constexpr int SMEM_USED = OFF_TMEMPTR + 16 + 1024;
  static constexpr int SMEM_BYTES = SMEM_USED > 119808 ? SMEM_USED : 119808;
};

// barrier indices
constexpr int kBarA = 0;      // K,V (dK/dV kernel) or Q,dO (dQ kernel): loaded once
constexpr int kBarB = 1;      // the per-iteration tile pair, buffers 0 and 1 (kBarB, kBarB + 1)
constexpr int kBarS = 3;      // both score products done
constexpr int kBarP = 4;      // every element-wise thread wrote its P / dS
constexpr int kBarO = 5;      // accumulation products done
constexpr int kBarRow = 6;    // dK/dV kernel: row data (D, lse) of even iterations staged
constexpr int kBarDrain = 7;
constexpr int kBarRow2 = 8;   // dK/dV kernel: row data of odd iterations staged
constexpr int kBarRead = 6;   // dQ kernel: every element-wise thread has read S and dP
constexpr int kBarKf = 8;     // dQ kernel: K buffers 0-2 loaded (kBarB, kBarB + 1: V buffers)

__device__ __forceinline__ bool bwd_wait(uint32_t bar, uint32_t parity, const PrefillArgs& a) {
  for (int i = 0; i < 256; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > a.timeout_ns) {
      atomicCAS(a.err, 0, kStatusTimeout);
      return false;
    }
  }
  return true;
}

// D_t = sum_c dO[t, c] O[t, c] for one row of d bf16 elements (fp32 accumulation).
template <int D>
__device__ __forceinline__ float row_dot(const __nv_bfloat16* x, const __nv_bfloat16* y) {
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < D; c += 8) {
    const uint4 u = *reinterpret_cast<const uint4*>(x + c);
    const uint4 w = *reinterpret_cast<const uint4*>(y + c);
    const uint32_t uu[4] = {u.x, u.y, u.z, u.w}, ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(__uint_as_float(uu[i] << 16), __uint_as_float(ww[i] << 16), acc);
      acc = fmaf(__uint_as_float(uu[i] & 0xffff0000u), __uint_as_float(ww[i] & 0xffff0000u), acc);
    }
  }
  return acc;
}

// Columns c in [0, 128) of a score tile whose absolute index lies in [lo, hi] or in
// [0, sk_hi], as four 32-bit words (bit c of word c / 32).
__device__ __forceinline__ void visible_words(int lo, int hi, int sk_hi, uint32_t* w) {
#pragma unroll
  for (int k = 0; k < 4; ++k) w[k] = range_bits(lo, hi, 32 * k) | range_bits(0, sk_hi, 32 * k);
}
__device__ __forceinline__ bool word_bit(const uint32_t* w, int c) {
  return static_cast<int>(w[c >> 5] << (31 - (c & 31))) < 0;
}

// TMEM column of K-step kk (16 score columns, 8 packed bf16 columns) of the packed
// P / dS operand.  Each warpgroup writes its 64 columns packed into the first 32 of
// the 64 it read (never into the other warpgroup's, which may still be unread):
// steps 0-3 at columns 0-31, steps 4-7 at 64-95.
__host__ __device__ constexpr uint32_t packed_col(int kk) { return kk * 8 + (kk >= 4 ? 32 : 0); }

// Element-wise step of the dK/dV kernel for one key row over 64 query columns
// col0 .. col0 + 63: P^T = exp2(S^T scale log2 e - lse log2 e) (zero where the pair
// is not visible, tested only when MASK), dS^T = P^T (dP^T - D); D and the log2 lse
// of the columns come from shared memory four at a time.  Packed bf16 pairs out.
template <bool MASK>
__device__ __forceinline__ void dkdv_elementwise(const uint32_t* sr, const uint32_t* dr, const float* D_s,
                                                 const float* L_s, float sl2, const uint32_t* vw, int col0,
                                                 uint32_t* pw, uint32_t* dw) {
#pragma unroll
  for (int c = 0; c < 64; c += 4) {
    const float4 l4 = *reinterpret_cast<const float4*>(L_s + col0 + c);
    const float4 d4 = *reinterpret_cast<const float4*>(D_s + col0 + c);
    const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w};
    float p[4], ds[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float pe = ex2_approx(fmaf(__uint_as_float(sr[c + e]), sl2, -lv[e]));
      if (MASK) pe = word_bit(vw, col0 + c + e) ? pe : 0.f;
      p[e] = pe;
      ds[e] = pe * (__uint_as_float(dr[c + e]) - dv[e]);
    }
    pw[c / 2] = pack_bf16x2(p[0], p[1]);
    pw[c / 2 + 1] = pack_bf16x2(p[2], p[3]);
    dw[c / 2] = pack_bf16x2(ds[0], ds[1]);
    dw[c / 2 + 1] = pack_bf16x2(ds[2], ds[3]);
  }
}

// Element-wise step of the dQ kernel for one query row (its D and log2 lse in
// registers) over 64 key columns col0 .. col0 + 63: dS = P (dP - D).
template <bool MASK>
__device__ __forceinline__ void dq_elementwise(const uint32_t* sr, const uint32_t* dr, float dt, float l2,
                                               float sl2, const uint32_t* vw, int col0, uint32_t* dw) {
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    float ds[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float pe = ex2_approx(fmaf(__uint_as_float(sr[c + e]), sl2, -l2));
      if (MASK) pe = word_bit(vw, col0 + c + e) ? pe : 0.f;
      ds[e] = pe * (__uint_as_float(dr[c + e]) - dt);
    }
    dw[c / 2] = pack_bf16x2(ds[0], ds[1]);
  }
}

template <int D>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar, int head, int row) {
#pragma unroll
  for (int c = 0; c < BwdCfg<D>::NCHUNK; ++c) tma_load_3d(dst + c * (kBM * 128), map, bar, c * 64, head, row);
}

// ------------------------------------------------------------------ D
// D[(b * Hq + h) * L + t] = rowsum(dout * out) of row (b, t, h), one thread per row.
template <int D>
__global__ void __launch_bounds__(256) swa_bwd_dot_kernel(const __grid_constant__ BwdArgs ba) {
  const PrefillArgs& a = ba.pa;
  const long long rows = static_cast<long long>(a.n_seq) * a.L * a.Hq;
  for (long long r = blockIdx.x * 256LL + threadIdx.x; r < rows; r += static_cast<long long>(gridDim.x) * 256) {
    const int h = static_cast<int>(r % a.Hq);
    const long long bt = r / a.Hq;
    const int t = static_cast<int>(bt % a.L);
    const long long b = bt / a.L;
    ba.dq[(b * a.Hq + h) * a.L + t] = row_dot<D>(static_cast<const __nv_bfloat16*>(ba.dout) + r * D,
                                                  static_cast<const __nv_bfloat16*>(ba.out) + r * D);
  }
}

// ------------------------------------------------------------------ dK, dV
// Roles (288 threads): warps 0-7 the element-wise step (warpgroup 0 on score
// columns 0-63, warpgroup 1 on 64-127; thread = TMEM lane = key row); warp 8 the
// producer, whose lane 0 issues the TMA loads and the MMAs and whose 32 lanes copy
// the per-row data (D and lse) into a two-slot staging buffer.  For iteration it
// the producer waits until every element-wise thread has written P^T(it) and
// dS^T(it), issues dV += P^T dO and dK += dS^T Q and right behind them S^T and dP^T
// of iteration it + 1 (the tensor pipe runs in issue order, so those overwrite P^T
// and dS^T only after the accumulation has read them), copies the row data of
// it + 2 into the slot iteration it has finished reading, publishes the row data
// of it + 1, and, once the accumulation of it is done reading Q and dO, requests the
// tiles of it + 2 into that buffer.  The element-wise warps wait only for their
// iteration's row data and scores.
constexpr int kDkdvThreads = 288;
constexpr int kDkdvProducerWarp = 8;

template <int D>
__global__ void __launch_bounds__(kDkdvThreads, 1)
    swa_bwd_dkdv_kernel(const __grid_constant__ BwdArgs ba, const __grid_constant__ CUtensorMap tq,
                        const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                        const __grid_constant__ CUtensorMap tdo) {
  using C = BwdCfg<D>;
  const PrefillArgs& a = ba.pa;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8 * i; };
  const uint32_t sK = base + C::OFF_T, sV = sK + C::TILE, sQ = sV + C::TILE, sdO = sQ + C::TILE;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(gbase + C::OFF_TMEMPTR);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  const int tiles = (a.L + kBM - 1) / kBM;
  const int jt = blockIdx.x % tiles;
  const int kvh = (blockIdx.x / tiles) % a.Hkv;
  const int b = blockIdx.x / (tiles * a.Hkv);
  const int j0 = jt * kBN;
  const int it_hi = j0 < a.n_sink ? tiles - 1
                                  : min(tiles - 1, (min(j0 + kBN - 1, a.L - 1) + a.window - 1) / kBM);

  if (tid == 0) {
    for (int i = 0; i < C::NBAR; ++i)
      mbar_init(bar(i), i == kBarP ? kEwThreads : (i == kBarRow || i == kBarRow2 ? 32 : 1));
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_ptr), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const size_t row_base = static_cast<size_t>(b) * a.L;

  // iterations: (query head g, query tile) flattened, query tiles fastest
  const int nq = it_hi - jt + 1;
  const int n_it = a.G * nq;
  auto it_head = [&](int i) { return kvh * a.G + i / nq; };
  auto it_row0 = [&](int i) { return (jt + i % nq) * kBM; };
  // staging slot i & 1 of the row data: D at floats 0..127, lse (log2 units) at 128..255
  auto row_bar = [&](int i) { return bar((i & 1) ? kBarRow2 : kBarRow); };
  bool ok = true;

  if (warp == kDkdvProducerWarp) {
    const float* d_rows = ba.dq;                      // D, written by the D kernel
    const uint32_t stg = smem_u32(gbase + C::OFF_STG);
    // lane l copies rows l, l + 32, l + 64, l + 96 of iteration i (zero past the end)
    auto stage_rows = [&](int i) {
      const int h = it_head(i), t0 = it_row0(i);
      const uint32_t dst = stg + (i & 1) * 1024;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int rr = lane + 32 * m, t = t0 + rr;
        const bool in = t < a.L;
        const size_t idx = (static_cast<size_t>(b) * a.Hq + h) * a.L + (in ? t : 0);
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst + rr * 4), "l"(d_rows + idx),
                     "r"(in ? 4u : 0u) : "memory");
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst + 512 + rr * 4), "l"(ba.lse + idx),
                     "r"(in ? 4u : 0u) : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // once this lane's copies of iteration i have landed: lse to log2 units, publish
    auto publish_rows = [&](int i) {
      float* l2 = reinterpret_cast<float*>(gbase + C::OFF_STG + (i & 1) * 1024) + 128;
#pragma unroll
      for (int m = 0; m < 4; ++m) l2[lane + 32 * m] *= 1.4426950408889634f;
      mbar_arrive(row_bar(i));
    };
    // one descriptor per operand array, stepped by offsets (buffer, k-step)
    const uint64_t dK0 = kmajor_desc<4>(sK, kBN, 0), dV0 = kmajor_desc<4>(sV, kBN, 0);
    const uint64_t dQ0 = kmajor_desc<4>(sQ, kBM, 0), ddO0 = kmajor_desc<4>(sdO, kBM, 0);
    const uint64_t vQ0 = v_desc<false, 16>(sQ, 0), vdO0 = v_desc<false, 16>(sdO, 0);
    auto load_qdo = [&](int i) {                      // lane 0: Q, dO of iteration i into buffer i & 1
      const int buf = i & 1;
      mbar_expect_tx(bar(kBarB + buf), 2 * C::TILE);
      load_tile<D>(sQ + 2 * buf * C::TILE, &tq, bar(kBarB + buf), it_head(i), static_cast<int>(row_base) + it_row0(i));
      load_tile<D>(sdO + 2 * buf * C::TILE, &tdo, bar(kBarB + buf), it_head(i), static_cast<int>(row_base) + it_row0(i));
    };
    auto scores = [&](int i) {                        // lane 0: S^T = K Q^T, dP^T = V dO^T of iteration i
      const uint32_t off = 2 * (i & 1) * C::TILE;
#pragma unroll
      for (int kk = 0; kk < C::QK_STEPS; ++kk)
        umma_ss<false>(tmem, desc_add(dK0, kmajor_off<4, kBN>(kk)), desc_add(dQ0, off + kmajor_off<4, kBM>(kk)),
                       C::IDESC_SS, kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < C::QK_STEPS; ++kk)
        umma_ss<false>(tmem + 128, desc_add(dV0, kmajor_off<4, kBN>(kk)), desc_add(ddO0, off + kmajor_off<4, kBM>(kk)),
                       C::IDESC_SS, kk > 0 ? 1u : 0u);
      tc_commit(bar(kBarS));
    };
    auto accumulate = [&](int i) {                    // lane 0: dV += P^T dO, dK += dS^T Q of iteration i
      const uint32_t off = 2 * (i & 1) * C::TILE;
#pragma unroll
      for (int kk = 0; kk < C::PV_STEPS; ++kk)
        umma_ts<false>(tmem + 256, tmem + packed_col(kk), desc_add(vdO0, off + mnmajor_off<16>(kk)), C::IDESC_ACC,
                       (i == 0 && kk == 0) ? 0u : 1u);
#pragma unroll
      for (int kk = 0; kk < C::PV_STEPS; ++kk)
        umma_ts<false>(tmem + 256 + D, tmem + 128 + packed_col(kk), desc_add(vQ0, off + mnmajor_off<16>(kk)),
                       C::IDESC_ACC, (i == 0 && kk == 0) ? 0u : 1u);
      tc_commit(bar(kBarO));
    };

    int issued = 0, waited = 0;                       // Q/dO loads requested / their arrivals seen
    if (lane == 0) {
      mbar_expect_tx(bar(kBarA), 2 * C::TILE);
      load_tile<D>(sK, &tk, bar(kBarA), kvh, static_cast<int>(row_base) + j0);
      load_tile<D>(sV, &tv, bar(kBarA), kvh, static_cast<int>(row_base) + j0);
      load_qdo(0);
      issued = 1;
      if (n_it > 1) {
        load_qdo(1);
        issued = 2;
      }
    }
    stage_rows(0);
    if (n_it > 1) {
      stage_rows(1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    publish_rows(0);
    if (lane == 0) {
      ok = bwd_wait(bar(kBarA), 0, a) && bwd_wait(bar(kBarB), 0, a);
      if (ok) {
        waited = 1;
        tc_fence_after();
        scores(0);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    for (int it = 0; ok && it < n_it; ++it) {
      // every element-wise thread has written P^T(it) and dS^T(it)
      if (!(ok = bwd_wait(bar(kBarP), it & 1, a))) break;
      if (lane == 0) {
        tc_fence_after();
        accumulate(it);
        if (it + 1 < n_it) {
          ok = bwd_wait(bar(kBarB + ((it + 1) & 1)), ((it + 1) >> 1) & 1, a);
          if (ok) {
            waited = it + 2;
            tc_fence_after();
            scores(it + 1);
          }
        }
      }
      if (!(ok = __shfl_sync(0xffffffffu, ok, 0))) break;
      // slot it & 1 is free (every thread is past iteration it): copy it + 2 into it
      if (it + 2 < n_it) {
        stage_rows(it + 2);
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      }
      if (it + 1 < n_it) publish_rows(it + 1);
      if (lane == 0 && it + 2 < n_it) {
        // the accumulation of it read Q and dO from buffer it & 1
        if ((ok = bwd_wait(bar(kBarO), it & 1, a))) {
          load_qdo(it + 2);
          issued = it + 3;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    if (lane == 0) {
      // Every product is issued: the drain barrier completes (its only phase) when all
      // have finished, which is when the element-wise warps read the accumulators.
      tc_commit(bar(kBarDrain));
      if (!ok) {
        // let everything this thread started finish before the CTA releases its memory
        bwd_wait(bar(kBarDrain), 0, a);
        bwd_wait(bar(kBarA), 0, a);
        for (int i = waited; i < issued; ++i) bwd_wait(bar(kBarB + (i & 1)), (i >> 1) & 1, a);
      }
    }
    __syncwarp();
  } else {
    const int r = tid & 127;                          // TMEM lane (key row) of this thread
    const int half = tid >> 7;                        // score columns 64 half .. 64 half + 63
    const uint32_t lane_off = static_cast<uint32_t>((r >> 5) * 32) << 16;
    const int s_key = j0 + r;                         // this thread's key (TMEM lane)
    // query rows that see this key: s_key .. s_key + window - 1 (all later rows for a
    // sink), before the sequence's end
    const int t_hi = min(a.L - 1, s_key < a.n_sink ? a.L - 1 : s_key + a.window - 1);
    for (int it = 0; it < n_it; ++it) {
      const int i0 = it_row0(it);
      if (!(ok = __all_sync(0xffffffffu, bwd_wait(row_bar(it), (it >> 1) & 1, a) &&
                                             bwd_wait(bar(kBarS), it & 1, a))))
        break;
      tc_fence_after();
      const float* D_s = reinterpret_cast<const float*>(gbase + C::OFF_STG + (it & 1) * 1024);
      const float* L_s = D_s + 128;
      // P^T and dS^T of this key row over this warpgroup's 64 query columns
      {
        // every (key, query) pair of the tile visible: no test per column
        const bool full = j0 + kBN - 1 <= i0 && i0 + kBM - 1 < a.L &&
                          (j0 >= i0 + kBM - a.window || j0 + kBN - 1 < a.n_sink);
        uint32_t sr[64], dr[64];
        tmem_ld64_wait(tmem + lane_off + 64 * half, sr);
        tmem_ld64_wait(tmem + lane_off + 128 + 64 * half, dr);
        uint32_t pw[32], dw[32];
        if (full) {
          dkdv_elementwise<false>(sr, dr, D_s, L_s, a.scale_log2, nullptr, 64 * half, pw, dw);
        } else {
          uint32_t vw[4];
          visible_words(s_key - i0, t_hi - i0, -1, vw);
          dkdv_elementwise<true>(sr, dr, D_s, L_s, a.scale_log2, vw, 64 * half, pw, dw);
        }
        // packed into the first half of this warpgroup's own columns: the other
        // warpgroup may still be reading its S^T and dP^T columns
        tmem_st32(tmem + lane_off + 64 * half, pw);
        tmem_st32(tmem + lane_off + 128 + 64 * half, dw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBarP));
    }
    // all products done (a single-phase barrier: no parity can be confused with another)
    ok = __all_sync(0xffffffffu, ok && bwd_wait(bar(kBarDrain), 0, a));
    tc_fence_after();
    if (ok) {                                 // warp-uniform: the TMEM loads are warp-collective
      const bool row_ok = s_key < a.L;
      float* dv = ba.dv + ((row_base + (row_ok ? s_key : 0)) * a.Hkv + kvh) * D;
      float* dk = ba.dk + ((row_base + (row_ok ? s_key : 0)) * a.Hkv + kvh) * D;
#pragma unroll 1
      for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {   // this warpgroup's half of d
        uint32_t rv[32], rk[32];
        tmem_ld32_wait(tmem + lane_off + 256 + 32 * c, rv);
        tmem_ld32_wait(tmem + lane_off + 256 + D + 32 * c, rk);
        if (!row_ok) continue;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          *reinterpret_cast<float4*>(dv + 32 * c + i) = make_float4(
              __uint_as_float(rv[i]), __uint_as_float(rv[i + 1]), __uint_as_float(rv[i + 2]), __uint_as_float(rv[i + 3]));
          *reinterpret_cast<float4*>(dk + 32 * c + i) =
              make_float4(__uint_as_float(rk[i]) * a.scale, __uint_as_float(rk[i + 1]) * a.scale,
                          __uint_as_float(rk[i + 2]) * a.scale, __uint_as_float(rk[i + 3]) * a.scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ dQ
// Roles as in the dK/dV kernel: warps 0-7 the element-wise step (thread = TMEM lane
// = query row, warpgroup 0 on key columns 0-63, warpgroup 1 on 64-127), warp 8
// (lane 0) TMA and MMA.  dS goes to TMEM columns 384-511, apart from S and dP, so
// the scores of key tile j + 1 are computed while the element-wise step of j runs:
// the element-wise warps signal once they have read S(j) and dP(j) (barrier R), the
// producer then issues S and dP of j + 1, and after dS(j) is written, dQ += dS K.
// An element-wise warp writes dS(j) only after the accumulation of j - 1 has read
// dS(j - 1).  K is kept in three buffers and V in two: V of tile j + 2 is requested
// as soon as the scores of j have been read, K of tile j + 3 once the accumulation
// of j has read K(j), so both arrive a key tile or more before their score products.
constexpr int kDqThreads = 288;
constexpr int kDqProducerWarp = 8;

template <int D>
__global__ void __launch_bounds__(kDqThreads, 1)
    swa_bwd_dq_kernel(const __grid_constant__ BwdArgs ba, const __grid_constant__ CUtensorMap tq,
                      const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                      const __grid_constant__ CUtensorMap tdo) {
  using C = DqCfg<D>;
  const PrefillArgs& a = ba.pa;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8 * i; };
  const uint32_t sQ = base + C::OFF_T, sdO = sQ + C::TILE, sK = base + C::OFF_K, sV = base + C::OFF_V;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(gbase + C::OFF_TMEMPTR);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  const int tiles = (a.L + kBM - 1) / kBM;
  const int qt = blockIdx.x % tiles;
  const int h = (blockIdx.x / tiles) % a.Hq;
  const int b = blockIdx.x / (tiles * a.Hq);
  const int kvh = h / a.G;
  Unit x;
  decode_tile(a, nullptr, nullptr, b * tiles + qt, x);

  if (tid == 0) {
    for (int i = 0; i < C::NBAR; ++i) mbar_init(bar(i), i == kBarP || i == kBarRead ? kEwThreads : 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_ptr), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const uint32_t tmem_ds = tmem + 384;                // packed dS (see packed_col)
  const size_t row_base = static_cast<size_t>(b) * a.L;
  const int n = x.n_tiles;
  bool ok = true;

  if (warp == kDqProducerWarp) {
    if (lane == 0) {
      // one descriptor per operand array, stepped by offsets (buffer, k-step)
      const uint64_t dQ0 = kmajor_desc<4>(sQ, kBM, 0), ddO0 = kmajor_desc<4>(sdO, kBM, 0);
      const uint64_t dK0 = kmajor_desc<4>(sK, kBN, 0), dV0 = kmajor_desc<4>(sV, kBN, 0);
      const uint64_t vK0 = v_desc<false, 16>(sK, 0);
      auto load_k = [&](int jj) {                     // K of key tile step jj into K buffer jj % 3
        const int buf = jj % 3;
        mbar_expect_tx(bar(kBarKf + buf), C::TILE);
        load_tile<D>(sK + buf * C::TILE, &tk, bar(kBarKf + buf), kvh, static_cast<int>(row_base) + tile_n0(x, jj));
      };
      auto load_v = [&](int jj) {                     // V of key tile step jj into V buffer jj & 1
        const int buf = jj & 1;
        mbar_expect_tx(bar(kBarB + buf), C::TILE);
        load_tile<D>(sV + buf * C::TILE, &tv, bar(kBarB + buf), kvh, static_cast<int>(row_base) + tile_n0(x, jj));
      };
      auto wait_k = [&](int jj) { return bwd_wait(bar(kBarKf + jj % 3), (jj / 3) & 1, a); };
      auto wait_v = [&](int jj) { return bwd_wait(bar(kBarB + (jj & 1)), (jj >> 1) & 1, a); };
      auto scores = [&](int jj) {                     // S = Q K^T, dP = dO V^T of key tile step jj
        const uint32_t offk = (jj % 3) * C::TILE, offv = (jj & 1) * C::TILE;
#pragma unroll
        for (int kk = 0; kk < C::QK_STEPS; ++kk)
          umma_ss<false>(tmem, desc_add(dQ0, kmajor_off<4, kBM>(kk)), desc_add(dK0, offk + kmajor_off<4, kBN>(kk)),
                         C::IDESC_SS, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < C::QK_STEPS; ++kk)
          umma_ss<false>(tmem + 128, desc_add(ddO0, kmajor_off<4, kBM>(kk)), desc_add(dV0, offv + kmajor_off<4, kBN>(kk)),
                         C::IDESC_SS, kk > 0 ? 1u : 0u);
        tc_commit(bar(kBarS));
      };
      auto accumulate = [&](int jj) {                 // dQ += dS K of key tile step jj
        const uint32_t offk = (jj % 3) * C::TILE;
#pragma unroll
        for (int kk = 0; kk < C::PV_STEPS; ++kk)
          umma_ts<false>(tmem + 256, tmem_ds + packed_col(kk), desc_add(vK0, offk + mnmajor_off<16>(kk)), C::IDESC_ACC,
                         (jj == 0 && kk == 0) ? 0u : 1u);
        tc_commit(bar(kBarO));
      };
      // loads requested / their arrivals seen, for K and for V
      int issued_k = 0, issued_v = 0, waited_k = 0, waited_v = 0;
      mbar_expect_tx(bar(kBarA), 2 * C::TILE);
      load_tile<D>(sQ, &tq, bar(kBarA), h, static_cast<int>(row_base) + x.m0);
      load_tile<D>(sdO, &tdo, bar(kBarA), h, static_cast<int>(row_base) + x.m0);
      for (; issued_k < min(n, 3); ++issued_k) load_k(issued_k);
      for (; issued_v < min(n, 2); ++issued_v) load_v(issued_v);
      if ((ok = bwd_wait(bar(kBarA), 0, a) && wait_k(0) && wait_v(0))) {
        waited_k = waited_v = 1;
        tc_fence_after();
        scores(0);
      }
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n) {
          // S(j) and dP(j) have been read, so the score products of j are done: V buffer
          // j & 1 takes V of j + 2, and the score columns take the scores of j + 1
          if (!(ok = bwd_wait(bar(kBarRead), j & 1, a))) break;
          if (j + 2 < n) {
            load_v(j + 2);
            issued_v = j + 3;
          }
          if (!(ok = wait_k(j + 1) && wait_v(j + 1))) break;
          waited_k = waited_v = j + 2;
          tc_fence_after();
          scores(j + 1);
        }
        if (!(ok = bwd_wait(bar(kBarP), j & 1, a))) break;      // dS(j) written
        tc_fence_after();
        accumulate(j);
        if (j + 3 < n) {
          // the accumulation of j is the last reader of K buffer j % 3
          if (!(ok = bwd_wait(bar(kBarO), j & 1, a))) break;
          load_k(j + 3);
          issued_k = j + 4;
        }
      }
      // every product is issued: the drain barrier's only phase completes when all are done
      tc_commit(bar(kBarDrain));
      if (!ok) {
        // let everything this thread started finish before the CTA releases its memory
        bwd_wait(bar(kBarDrain), 0, a);
        bwd_wait(bar(kBarA), 0, a);
        for (int i = waited_k; i < issued_k; ++i) wait_k(i);
        for (int i = waited_v; i < issued_v; ++i) wait_v(i);
      }
    }
    __syncwarp();
  } else {
    const int r = tid & 127;                          // TMEM lane (query row) of this thread
    const int half = tid >> 7;                        // key columns 64 half .. 64 half + 63
    const uint32_t lane_off = static_cast<uint32_t>((r >> 5) * 32) << 16;
    const int t = x.m0 + r;                           // this thread's query row
    float dt = 0.f, l2 = 0.f;
    if (t < a.L) {
      const size_t off = ((row_base + t) * a.Hq + h) * D;
      dt = row_dot<D>(static_cast<const __nv_bfloat16*>(ba.dout) + off, static_cast<const __nv_bfloat16*>(ba.out) + off);
      l2 = ba.lse[(static_cast<size_t>(b) * a.Hq + h) * a.L + t] * 1.4426950408889634f;
    }
    for (int j = 0; j < n; ++j) {
      const int n0 = tile_n0(x, j);
      if (!(ok = __all_sync(0xffffffffu, bwd_wait(bar(kBarS), j & 1, a)))) break;
      tc_fence_after();
      // dS of this query row over this warpgroup's 64 key columns, written over S
      {
        uint32_t sr[64], dr[64];
        tmem_ld64_wait(tmem + lane_off + 64 * half, sr);
        tmem_ld64_wait(tmem + lane_off + 128 + 64 * half, dr);
        tc_fence_before();
        mbar_arrive(bar(kBarRead));                   // S(j), dP(j) read
        uint32_t dw[32];
        if (tile_needs_mask(x, j, a.window) || x.m1 - x.m0 != kBM - 1) {
          // keys t - window + 1 .. t and the sinks below min(n_sink, t + 1); nothing past the end
          uint32_t vw[4] = {0u, 0u, 0u, 0u};
          if (t < a.L) visible_words(t - a.window + 1 - n0, t - n0, min(a.n_sink, t + 1) - 1 - n0, vw);
          dq_elementwise<true>(sr, dr, dt, l2, a.scale_log2, vw, 64 * half, dw);
        } else {
          dq_elementwise<false>(sr, dr, dt, l2, a.scale_log2, nullptr, 64 * half, dw);
        }
        // the accumulation of j - 1 has read dS(j - 1) before it is overwritten
        if (j > 0 && !(ok = __all_sync(0xffffffffu, bwd_wait(bar(kBarO), (j - 1) & 1, a)))) break;
        tc_fence_after();
        tmem_st32(tmem_ds + lane_off + 64 * half, dw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBarP));
    }
    // all products done (a single-phase barrier: no parity can be confused with another)
    ok = __all_sync(0xffffffffu, ok && bwd_wait(bar(kBarDrain), 0, a));
    tc_fence_after();
    if (ok) {                                 // warp-uniform: the TMEM loads are warp-collective
      const bool row_ok = t < a.L;
      float* dq = ba.dq + ((row_base + (row_ok ? t : 0)) * a.Hq + h) * D;
#pragma unroll 1
      for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {   // this warpgroup's half of d
        uint32_t rr[32];
        tmem_ld32_wait(tmem + lane_off + 256 + 32 * c, rr);
        if (!row_ok) continue;
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(dq + 32 * c + i) =
              make_float4(__uint_as_float(rr[i]) * a.scale, __uint_as_float(rr[i + 1]) * a.scale,
                          __uint_as_float(rr[i + 2]) * a.scale, __uint_as_float(rr[i + 3]) * a.scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int D>
cudaError_t launch_bwd_impl(const BwdArgs& ba, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, const CUtensorMap& tdo, cudaStream_t stream) {
  using C = BwdCfg<D>;
  const PrefillArgs& a = ba.pa;
  const long long tiles = (a.L + kBM - 1) / kBM;
  const long long g_kv = tiles * a.Hkv * a.n_seq, g_q = tiles * a.Hq * a.n_seq;
  if (g_kv == 0) return cudaSuccess;
  if (g_q > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(swa_bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  static_assert(DqCfg<D>::SMEM_BYTES <= 232448, "shared memory budget");
  e = cudaFuncSetAttribute(swa_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, DqCfg<D>::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // one CTA per SM (see SMEM_BYTES): refuse to launch if the occupancy says otherwise
  static int checked = 0;
  if (!checked) {
    int n1 = 0, n2 = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n1, swa_bwd_dkdv_kernel<D>, kDkdvThreads, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n2, swa_bwd_dq_kernel<D>, kDqThreads, DqCfg<D>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (n1 != 1 || n2 != 1) return cudaErrorNotSupported;
    checked = 1;
  }
  const long long rows = static_cast<long long>(a.n_seq) * a.L * a.Hq;
  swa_bwd_dot_kernel<D><<<static_cast<unsigned>(std::min<long long>((rows + 255) / 256, 148LL * 32)), 256, 0, stream>>>(ba);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  swa_bwd_dkdv_kernel<D><<<static_cast<unsigned>(g_kv), kDkdvThreads, C::SMEM_BYTES, stream>>>(ba, tq, tk, tv, tdo);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  swa_bwd_dq_kernel<D><<<static_cast<unsigned>(g_q), kDqThreads, DqCfg<D>::SMEM_BYTES, stream>>>(ba, tq, tk, tv, tdo);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(const BwdArgs& ba, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, int d, cudaStream_t stream) {
  if (d == 64) return launch_bwd_impl<64>(ba, tq, tk, tv, tdo, stream);
  if (d == 128) return launch_bwd_impl<128>(ba, tq, tk, tv, tdo, stream);
  return cudaErrorInvalidValue;
}

}  // namespace swa
