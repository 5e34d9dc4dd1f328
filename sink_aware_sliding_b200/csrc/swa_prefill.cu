// Prefill of causal sliding-window attention with attention sinks on sm_100a.
//
// Operation ("Sliding-window beats linear attention", sections 1 and 3): row t
// attends to keys j <= t with j >= t - window + 1 or j < n_sink.
//
// One persistent CTA per SM walks work units (sequence, query head, 128-row
// query tile).  Per unit only the key tiles that can hold a visible key are
// visited: the band tiles covering [m0 - window + 1, m0 + 127] and, when the
// band has moved past them, the tiles holding the sink prefix.  Everything
// else is never loaded and never multiplied.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r.  Loads S from
//              tensor memory, masks edge tiles, runs the online softmax in
//              fp32 (exp2 with log2(e) folded into the scale, rescale of O only
//              when the running max grows by more than 2^8), writes P over S
//              in tensor memory, and finally normalises O and stores O and LSE.
//   warp 4     TMA: Q tile (double-buffered across units) and K/V tiles
//              (NSTAGE-deep ring) with 128-byte swizzle.
//   warp 5     MMA: one thread issues tcgen05.mma.  S = Q K^T into one of two
//              TMEM S buffers, then O += P V with P read from TMEM.  S(g+1) is
//              issued before O += P(g) V so the tensor pipe works while the
//              softmax warps handle tile g.
// Every barrier wait is bounded by a time limit; on expiry the CTA records
// SWA_ERR_DEVICE_TIMEOUT, stops issuing work, drains what it issued, frees its
// tensor memory and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

#include "ptx.cuh"
#include "swa_internal.h"

namespace swa {
namespace {

constexpr int kThreads = 192;
constexpr int kSoftmaxThreads = 128;
constexpr int kLoadWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kStatusTimeout = 4;  // SWA_ERR_DEVICE_TIMEOUT

template <int D, bool F32>
struct Cfg {
  static constexpr int ELEM = F32 ? 4 : 2;
  static constexpr int CHUNK = 128 / ELEM;        // elements in one 128-byte swizzled row
  static constexpr int NCHUNK = D / CHUNK;
  static constexpr int KSTEP = 32 / ELEM;         // K of one MMA instruction (32 bytes)
  static constexpr int QK_STEPS = D / KSTEP;
  static constexpr int PV_STEPS = kBN / KSTEP;
  static constexpr int Q_BYTES = kBM * D * ELEM;
  static constexpr int KV_BYTES = kBN * D * ELEM;
  static constexpr int NSTAGE = (KV_BYTES <= 16384) ? 4 : 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NSTAGE * KV_BYTES;
  static constexpr int OFF_MISC = OFF_V + NSTAGE * KV_BYTES;
  // barriers: q_full[2] q_empty[2] k_full[NS] v_full[NS] kv_empty[NS] s_full[2] p_full[2]
  //           o_done o_final drain
  static constexpr int NBAR = 2 + 2 + 3 * NSTAGE + 2 + 2 + 3;
  static constexpr int OFF_TABLES = OFF_MISC + 8 * NBAR + 16;   // + tmem base + abort flag
  static constexpr int SMEM_BYTES = OFF_TABLES + 2 * 4 * (kMaxSeqSmem + 1) + 1024;  // +align slack
  static constexpr uint32_t IDESC_QK = make_idesc(F32 ? 2u : 1u, kBM, kBN, false);
  static constexpr uint32_t IDESC_PV = make_idesc(F32 ? 2u : 1u, kBM, D, true);
  static constexpr uint32_t TMEM_S0 = 0, TMEM_S1 = 128, TMEM_O = 256, TMEM_COLS = 512;
};

struct Unit {
  int seq, seq_start, len, m0, m1, h, kvh, nst, kb_lo, n_tiles;
};

struct Shared {
  uint32_t base;  // shared-space address of the aligned region
  uint32_t q_full[2], q_empty[2], s_full[2], p_full[2], o_done, o_final, drain;
  uint32_t k_full[4], v_full[4], kv_empty[4];
  volatile int* abort_flag;
  uint32_t* tmem_base;
  int* s_cu;    // varlen: cu_seqlens copy
  int* s_tpre;  // varlen: query tiles before each sequence
};

__device__ __forceinline__ void fail(const PrefillArgs& a, const Shared& sh) {
  *sh.abort_flag = 1;
  atomicCAS(a.err, 0, kStatusTimeout);
}

// Bounded wait on (bar, parity).  Returns false if the time limit ran out
// (which starts the CTA's abort) or, when honor_abort is set, as soon as
// another thread has started it.  Teardown waits pass honor_abort = false.
__device__ __noinline__ bool wait_bar(uint32_t bar, uint32_t parity, const PrefillArgs& a,
                                      const Shared& sh, bool honor_abort = true) {
  for (int i = 0; i < 256; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (honor_abort && *sh.abort_flag) return false;
    if (globaltimer_ns() - t0 > a.timeout_ns) {
      fail(a, sh);
      return false;
    }
  }
}

__device__ __forceinline__ bool get_unit(const PrefillArgs& a, const Shared& sh, int total_tiles,
                                         int u, Unit& x) {
  const int gt = total_tiles - 1 - u / a.Hq;  // heaviest (latest) tiles first
  x.h = u % a.Hq;
  x.kvh = x.h / a.G;
  int qt;
  if (a.cu_seqlens == nullptr) {
    const int tps = (a.L + kBM - 1) / kBM;
    x.seq = gt / tps;
    qt = gt - x.seq * tps;
    x.seq_start = x.seq * a.L;
    x.len = a.L;
  } else {
    int lo = 0, hi = a.n_seq - 1;  // last seq with s_tpre[seq] <= gt
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sh.s_tpre[mid] <= gt) lo = mid; else hi = mid - 1;
    }
    x.seq = lo;
    qt = gt - sh.s_tpre[lo];
    x.seq_start = sh.s_cu[lo];
    x.len = sh.s_cu[lo + 1] - sh.s_cu[lo];
  }
  x.m0 = qt * kBM;
  x.m1 = min(x.m0 + kBM, x.len) - 1;
  const int lo_key = max(0, x.m0 - a.window + 1);
  x.kb_lo = lo_key / kBN;
  const int kb_hi = x.m1 / kBN;
  x.nst = a.n_sink > 0 ? min((a.n_sink + kBN - 1) / kBN, x.kb_lo) : 0;
  x.n_tiles = x.nst + kb_hi - x.kb_lo + 1;
  return x.len > 0 && x.m0 < x.len;
}

__device__ __forceinline__ int tile_n0(const Unit& x, int j) {
  return (j < x.nst ? j : x.kb_lo + (j - x.nst)) * kBN;
}

template <int D, bool F32, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1)
    swa_prefill_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ CUtensorMap tq,
                       const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv) {
  using C = Cfg<D, F32>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  Shared sh;
  sh.base = base;
  {
    uint32_t b = base + C::OFF_MISC;
    auto next = [&]() { uint32_t r = b; b += 8; return r; };
    sh.q_full[0] = next(); sh.q_full[1] = next();
    sh.q_empty[0] = next(); sh.q_empty[1] = next();
    for (int i = 0; i < C::NSTAGE; ++i) sh.k_full[i] = next();
    for (int i = 0; i < C::NSTAGE; ++i) sh.v_full[i] = next();
    for (int i = 0; i < C::NSTAGE; ++i) sh.kv_empty[i] = next();
    sh.s_full[0] = next(); sh.s_full[1] = next();
    sh.p_full[0] = next(); sh.p_full[1] = next();
    sh.o_done = next();
    sh.o_final = next();
    sh.drain = next();
    sh.tmem_base = reinterpret_cast<uint32_t*>(gbase + C::OFF_MISC + 8 * C::NBAR);
    sh.abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 8 * C::NBAR + 4);
    sh.s_cu = reinterpret_cast<int*>(gbase + C::OFF_TABLES);
    sh.s_tpre = sh.s_cu + (kMaxSeqSmem + 1);
  }
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    mbar_init(sh.q_full[0], 1); mbar_init(sh.q_full[1], 1);
    mbar_init(sh.q_empty[0], 1); mbar_init(sh.q_empty[1], 1);
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(sh.k_full[i], 1);
      mbar_init(sh.v_full[i], 1);
      mbar_init(sh.kv_empty[i], 1);
    }
    mbar_init(sh.s_full[0], 1); mbar_init(sh.s_full[1], 1);
    mbar_init(sh.p_full[0], kSoftmaxThreads); mbar_init(sh.p_full[1], kSoftmaxThreads);
    mbar_init(sh.o_done, 1);
    mbar_init(sh.o_final, 1);
    mbar_init(sh.drain, 1);
    *sh.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
  }
  // Varlen tables: copy cu_seqlens and prefix-sum the query tiles per sequence (warp 0).
  int total_tiles = a.total_tiles;
  if (a.cu_seqlens != nullptr) {
    if (warp == 0) {
      const int n = a.n_seq;
      const int per = (n + 31) / 32;
      int local = 0;
      for (int i = lane * per; i < min(n, (lane + 1) * per); ++i) {
        const int c0 = a.cu_seqlens[i], c1 = a.cu_seqlens[i + 1];
        sh.s_cu[i] = c0;
        local += (c1 - c0 + kBM - 1) / kBM;
      }
      if (lane == 0) sh.s_cu[n] = a.cu_seqlens[n];
      int incl = local;
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      int run = incl - local;
      for (int i = lane * per; i < min(n, (lane + 1) * per); ++i) {
        sh.s_tpre[i] = run;
        run += (a.cu_seqlens[i + 1] - a.cu_seqlens[i] + kBM - 1) / kBM;
      }
      if (lane == 31) sh.s_tpre[n] = incl;
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(sh.tmem_base), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (a.cu_seqlens != nullptr) total_tiles = sh.s_tpre[a.n_seq];
  const uint32_t tmem = *sh.tmem_base;
  const int n_units = total_tiles * a.Hq;

  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int g = 0, uc = 0;
      int last_g[4] = {-1, -1, -1, -1};
      int last_q[2] = {-1, -1};
      const bool skip = (a.debug_flags & 1) != 0;
      bool ok = !skip;
      for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++uc) {
        Unit x;
        if (!get_unit(a, sh, total_tiles, u, x)) continue;
        const int qb = uc & 1;
        if (!(ok = wait_bar(sh.q_empty[qb], ((uc >> 1) & 1) ^ 1, a, sh))) break;
        mbar_expect_tx(sh.q_full[qb], C::Q_BYTES);
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_3d(base + C::OFF_Q + qb * C::Q_BYTES + c * (kBM * 128), &tq, sh.q_full[qb],
                      c * C::CHUNK, x.h, x.seq_start + x.m0);
        last_q[qb] = uc;
        for (int j = 0; j < x.n_tiles; ++j, ++g) {
          const int st = g % C::NSTAGE;
          if (!(ok = wait_bar(sh.kv_empty[st], ((g / C::NSTAGE) & 1) ^ 1, a, sh))) break;
          const int row = x.seq_start + tile_n0(x, j);
          mbar_expect_tx(sh.k_full[st], C::KV_BYTES);
          for (int c = 0; c < C::NCHUNK; ++c)
            tma_load_3d(base + C::OFF_K + st * C::KV_BYTES + c * (kBN * 128), &tk, sh.k_full[st],
                        c * C::CHUNK, x.kvh, row);
          mbar_expect_tx(sh.v_full[st], C::KV_BYTES);
          for (int c = 0; c < C::NCHUNK; ++c)
            tma_load_3d(base + C::OFF_V + st * C::KV_BYTES + c * (kBN * 128), &tv, sh.v_full[st],
                        c * C::CHUNK, x.kvh, row);
          last_g[st] = g;
        }
      }
      if (*sh.abort_flag) {
        // Let copies already in flight land before the CTA exits.
        for (int st = 0; st < C::NSTAGE; ++st)
          if (last_g[st] >= 0) {
            const uint32_t ph = (last_g[st] / C::NSTAGE) & 1;
            wait_bar(sh.k_full[st], ph, a, sh, false);
            wait_bar(sh.v_full[st], ph, a, sh, false);
          }
        for (int qb = 0; qb < 2; ++qb)
          if (last_q[qb] >= 0) wait_bar(sh.q_full[qb], (last_q[qb] >> 1) & 1, a, sh, false);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int g = 0, uc = 0;
      int prev_g = -1;
      bool prev_first = false, prev_last = false;
      bool ok = true;
      auto issue_pv = [&](int pg, bool first, bool last) -> bool {
        const int st = pg % C::NSTAGE;
        if (!wait_bar(sh.p_full[pg & 1], (pg >> 1) & 1, a, sh)) return false;
        if (!wait_bar(sh.v_full[st], (pg / C::NSTAGE) & 1, a, sh)) return false;
        tc_fence_after();
        const uint32_t p_tmem = tmem + ((pg & 1) ? C::TMEM_S1 : C::TMEM_S0);
        const uint32_t v_base = base + C::OFF_V + st * C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::PV_STEPS; ++kk) {
          // B = V (MN-major): K-step = KSTEP key rows of 128 bytes; LBO jumps between
          // 128-byte column chunks of d (kBN rows apart), SBO between swizzle atoms along
          // the keys (8 rows with the 128-byte swizzle; tf32 operands in MN-major order
          // need the 128-byte swizzle with 32-byte atoms, whose atom is 4 rows).
          const uint64_t bdesc =
              F32 ? smem_desc(v_base + kk * (C::KSTEP * 128), kBN * 128, 512, kLayoutSw128Atom32)
                  : smem_desc(v_base + kk * (C::KSTEP * 128), kBN * 128, 1024, kLayoutSw128);
          umma_ts<F32>(tmem + C::TMEM_O, p_tmem + kk * 8, bdesc, C::IDESC_PV,
                       (first && kk == 0) ? 0u : 1u);
        }
        tc_commit(sh.kv_empty[st]);
        tc_commit(sh.o_done);
        if (last) tc_commit(sh.o_final);  // O of the unit is complete
        return true;
      };
      for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++uc) {
        Unit x;
        if (!get_unit(a, sh, total_tiles, u, x)) continue;
        const int qb = uc & 1;
        if (!(ok = wait_bar(sh.q_full[qb], (uc >> 1) & 1, a, sh))) break;
        const uint32_t q_base = base + C::OFF_Q + qb * C::Q_BYTES;
        for (int j = 0; j < x.n_tiles; ++j, ++g) {
          const int st = g % C::NSTAGE;
          if (!(ok = wait_bar(sh.k_full[st], (g / C::NSTAGE) & 1, a, sh))) break;
          tc_fence_after();
          const uint32_t s_tmem = tmem + ((g & 1) ? C::TMEM_S1 : C::TMEM_S0);
          const uint32_t k_base = base + C::OFF_K + st * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::QK_STEPS; ++kk) {
            // A = Q, B = K (both K-major): 32-byte steps inside a 128-byte swizzled
            // row, next column chunk kBM (kBN) rows further on.
            const int ch = kk / (C::QK_STEPS / C::NCHUNK);
            const int wi = kk % (C::QK_STEPS / C::NCHUNK);
            const uint64_t adesc = smem_desc(q_base + ch * (kBM * 128) + wi * 32, 16, 1024, kLayoutSw128);
            const uint64_t bdesc = smem_desc(k_base + ch * (kBN * 128) + wi * 32, 16, 1024, kLayoutSw128);
            umma_ss<F32>(s_tmem, adesc, bdesc, C::IDESC_QK, kk > 0 ? 1u : 0u);
          }
          tc_commit(sh.s_full[g & 1]);
          if (j == x.n_tiles - 1) tc_commit(sh.q_empty[qb]);
          if (prev_g >= 0 && !(ok = issue_pv(prev_g, prev_first, prev_last))) break;
          prev_g = g;
          prev_first = (j == 0);
          prev_last = (j == x.n_tiles - 1);
        }
      }
      if (ok && prev_g >= 0) ok = issue_pv(prev_g, prev_first, prev_last);
      if (*sh.abort_flag) {
        // Wait until every MMA this thread issued has finished before TMEM is freed.
        tc_commit(sh.drain);
        wait_bar(sh.drain, 0, a, sh, false);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps
    const int r = tid;                                 // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    int g = 0, uc = 0, done_units = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++uc) {
      Unit x;
      if (!get_unit(a, sh, total_tiles, u, x)) continue;
      const int t = x.m0 + r;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < x.n_tiles; ++j, ++g) {
        ok = __all_sync(0xffffffffu, wait_bar(sh.s_full[g & 1], (g >> 1) & 1, a, sh));
        if (!ok) break;
        tc_fence_after();
        const uint32_t s_tmem = tmem + ((g & 1) ? C::TMEM_S1 : C::TMEM_S0) + lane_off;
        float s[kBN];
        {
          uint32_t sr[kBN];
          tmem_ld128_wait(s_tmem, sr);
#pragma unroll
          for (int i = 0; i < kBN; ++i) s[i] = __uint_as_float(sr[i]);
        }
        const int n0 = tile_n0(x, j);
        const bool need_mask = (j < x.nst) || (n0 + kBN - 1 > x.m0) || (n0 < x.m1 - a.window + 1);
        if (need_mask) {
          const int hi = t - n0;                    // visible: c <= hi
          const int lo = t - a.window + 1 - n0;     //   and (c >= lo
          const int sk = a.n_sink - n0;             //        or c < sk)
#pragma unroll
          for (int c = 0; c < kBN; ++c) {
            const bool vis = (c <= hi) && (c >= lo || c < sk);
            s[c] = vis ? s[c] : -INFINITY;
          }
        }
        float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
        for (int c = 4; c < kBN; c += 4) {
          mx0 = fmaxf(mx0, s[c]);
          mx1 = fmaxf(mx1, s[c + 1]);
          mx2 = fmaxf(mx2, s[c + 2]);
          mx3 = fmaxf(mx3, s[c + 3]);
        }
        const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        const float m_new = fmaxf(m_run, mx);
        // Move the reference max only when it grew by more than 2^8 in exp2 units
        // (NaN from -inf - -inf compares false: a fully masked row keeps -inf).
        const bool need = (m_new - m_run) * sl2 > 8.0f;
        const float m_use = need ? m_new : m_run;
        const float alpha = need ? ex2_approx((m_run - m_new) * sl2) : 1.0f;
        const float neg = (m_use == -INFINITY) ? 0.0f : -m_use * sl2;
        float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
        for (int c = 0; c < kBN; c += 2) {
          s[c] = ex2_approx(fmaf(s[c], sl2, neg));
          s[c + 1] = ex2_approx(fmaf(s[c + 1], sl2, neg));
          sum0 += s[c];
          sum1 += s[c + 1];
        }
        l_run = l_run * alpha + (sum0 + sum1);
        m_run = m_use;
        // P over S: bf16 pairs (element 2i in the low half of column i), or fp32.
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
        // Rescale O (rows of this warp) if any row moved its reference max.
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          ok = __all_sync(0xffffffffu, wait_bar(sh.o_done, (g - 1) & 1, a, sh));
          if (!ok) break;
          tc_fence_after();
          const uint32_t o_tmem = tmem + C::TMEM_O + lane_off;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t rr[32];
            tmem_ld32_wait(o_tmem + c * 32, rr);
#pragma unroll
            for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
            tmem_st32(o_tmem + c * 32, rr);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(sh.p_full[g & 1]);
      }
      if (!ok) break;
      // ---- epilogue: O / l -> out, LSE.  o_final completes once per unit, so its
      // parity is unambiguous here (o_done may lag two P.V products behind).
      ok = __all_sync(0xffffffffu, wait_bar(sh.o_final, done_units & 1, a, sh));
      if (!ok) break;
      ++done_units;
      tc_fence_after();
      const bool valid = t < x.len;
      const float inv_l = 1.0f / l_run;
      const uint32_t o_tmem = tmem + C::TMEM_O + lane_off;
      const size_t row = static_cast<size_t>(x.seq_start) + static_cast<size_t>(t);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32_wait(o_tmem + c * 32, rr);
        if (valid) {
          if constexpr (OUT_F32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) +
                                                    (row * a.Hq + x.h) * D + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(rr[4 * i]) * inv_l, __uint_as_float(rr[4 * i + 1]) * inv_l,
                                   __uint_as_float(rr[4 * i + 2]) * inv_l, __uint_as_float(rr[4 * i + 3]) * inv_l);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) +
                                                  (row * a.Hq + x.h) * D + c * 32);
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
      }
      if (valid && a.lse != nullptr) {
        const float ref = (m_run == -INFINITY) ? 0.0f : m_run * sl2;
        const float lse = (ref + log2f(l_run)) * 0.69314718055994531f;
        const size_t idx = a.lse_varlen
                               ? static_cast<size_t>(x.h) * static_cast<size_t>(a.T) + row
                               : (static_cast<size_t>(x.seq) * a.Hq + x.h) * a.L + t;
        a.lse[idx] = lse;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int D, bool F32, bool OUT_F32>
cudaError_t launch_impl(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                        const CUtensorMap& tv, int grid, cudaStream_t stream) {
  using C = Cfg<D, F32>;
  static_assert(C::SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(OUT_F32 || !F32, "fp32 inputs give fp32 outputs");
  auto kern = swa_prefill_kernel<D, F32, OUT_F32>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(a, tq, tk, tv);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tv, int d, bool f32, bool out_f32, int grid,
                           cudaStream_t stream) {
  if (f32) {
    if (d == 64) return launch_impl<64, true, true>(a, tq, tk, tv, grid, stream);
    return cudaErrorInvalidValue;
  }
  if (out_f32) {
    if (d == 64) return launch_impl<64, false, true>(a, tq, tk, tv, grid, stream);
    if (d == 128) return launch_impl<128, false, true>(a, tq, tk, tv, grid, stream);
    return cudaErrorInvalidValue;
  }
  if (d == 64) return launch_impl<64, false, false>(a, tq, tk, tv, grid, stream);
  if (d == 128) return launch_impl<128, false, false>(a, tq, tk, tv, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace swa
