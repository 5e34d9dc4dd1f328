// Prefill for short windows, sm_100a: d = 64, bf16 inputs, window <= 129 and no
// sink prefix, so a 128-row query tile m sees only key tiles m-1 and m (the
// sliding-window branch of a Based-style hybrid: "Simple linear attention
// language models balance the recall-throughput tradeoff", proposed method,
// windows of 64 or 128 tokens).
//
// With two key tiles per query tile, a per-unit pipeline (load Q and the band,
// two softmax steps, epilogue) spends most of its time starting and draining.
// Here a CTA streams a contiguous range of query tiles in (head, sequence, tile)
// order instead.  Consecutive query tiles of one sequence share a key tile, so
// each key tile is loaded once and serves both; the two softmax warpgroups take
// alternate query tiles and run independently, so one tile's softmax and
// epilogue overlap the other's.
//
// The products run on 64-key sub-tiles (halves of the 128-key tiles in shared
// memory, addressed by descriptor offsets).  Each warpgroup's 128-column S region
// holds two sub-tiles' S: the P of sub-tile g (packed bf16) occupies the first 32
// columns of its half, so S of sub-tile g+1 is computed into the other half while
// the warpgroup works on g, and the softmax finds its next S ready instead of
// waiting for P V -> Q K^T to round-trip.  A warp none of whose rows sees any key
// of a sub-tile skips it (with a 128-key window every warp skips one of the four
// sub-tiles of a query tile).
//
// Roles (384 threads):
//   warps 0-3   softmax + epilogue of the even query tiles of the range (A)
//   warps 4-7   the odd ones (B)
//   warp 8      TMA: per query tile its Q tile (4-slot ring) and the key tiles
//               not loaded yet, K and V of a key tile in one slot (4-slot ring)
//   warps 9, 10 tcgen05.mma issue, one thread for each softmax warpgroup (warp 9
//               also allocates TMEM): a tcgen05.mma issue stalls while the tensor
//               pipe is backed up, so one issuer per warpgroup keeps either from
//               waiting on the other's issue.  Per sub-tile g it issues S(g+1)
//               (into the half P(g-1) has left), waits for P(g), then O += P(g) V.
// A key-tile slot is freed after two arrivals: one commit per query tile that
// used it, plus an immediate arrive when only one query tile of the range uses
// it (the first tile of a range, or the last tile of a sequence).
// Barriers per warpgroup: S ready and P written, one per S half (so no wait can
// confuse two completed phases); a P V done barrier that the softmax waits on
// only to rescale O (S(g) ready implies P V of g-2 has finished, so that wait is
// unambiguous too); O final, one per O buffer.
// TMEM columns: S_A 0-127, S_B 128-255, then two O buffers per warpgroup (64
// columns each: O_A 256/320, O_B 384/448).  Query tile k of a warpgroup
// accumulates into buffer k mod 2, so the warpgroup writes out tile k-1 (its
// epilogue) while the tensor pipe computes tile k.
// With bf16 output, a finished query tile's Q slot is its output staging tile
// (TMA store), as in the pair kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "prefill_common.cuh"

namespace swa {
namespace {

using namespace prefill;

constexpr int kStreamThreads = 384;
constexpr int kStreamLoadWarp = 8;
constexpr int kStreamMmaWarp = 9;
// Same register split as the pair kernel: 168 at launch, 88 for the load/MMA
// warpgroup, 208 for the softmax warpgroups (2 * 128 * 208 + 128 * 88 = 384 * 168).
constexpr int kStreamLaunchRegs = 168;
constexpr uint32_t kStreamSoftmaxRegs = 208;
constexpr uint32_t kStreamProducerRegs = 88;
static_assert(2 * 128 * kStreamSoftmaxRegs + 128 * kStreamProducerRegs == kStreamThreads * kStreamLaunchRegs,
              "register split must use exactly the registers the block is launched with");

struct StreamCfg {
  static constexpr int D = 64;
  static constexpr int TILE = kBM * D * 2;          // one Q, K or V tile: 16 KB
  static constexpr int NQ = 4;                      // Q ring
  static constexpr int NKV = 4;                     // key-tile ring (K and V per slot)
  static constexpr int KSTEP = 16;                  // K of one bf16 MMA (32 bytes)
  static constexpr int QK_STEPS = D / KSTEP;
  static constexpr int SUB = 64;                    // keys per sub-tile (half a key tile)
  static constexpr int PV_STEPS = SUB / KSTEP;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + NQ * TILE;
  static constexpr int OFF_BAR = OFF_KV + NKV * 2 * TILE;
  static constexpr int B_QFULL = 0, B_QEMPTY = NQ, B_KVFULL = 2 * NQ, B_KVEMPTY = 2 * NQ + NKV,
                       B_SFULL = 2 * NQ + 2 * NKV, B_PFULL = B_SFULL + 4, B_PVDONE = B_PFULL + 4,
                       B_OFINAL = B_PVDONE + 2, B_DRAIN = B_OFINAL + 4, NBAR = B_DRAIN + 2;
  static constexpr int OFF_TMEMPTR = OFF_BAR + 8 * NBAR;
  static constexpr int OFF_ABORT = OFF_TMEMPTR + 4;
  static constexpr int OFF_TABLES = OFF_ABORT + 12;
  static constexpr int SMEM_BYTES = OFF_TABLES + 2 * 4 * (kMaxSeqSmem + 1) + 1024;
  static constexpr uint32_t IDESC_QK = make_idesc(1u, kBM, SUB, false);
  static constexpr uint32_t IDESC_PV = make_idesc(1u, kBM, D, true);
  __device__ static constexpr uint32_t tmem_s(int x) { return x ? 128u : 0u; }
  __device__ static constexpr uint32_t tmem_o(int x, int ob) { return 256u + 2 * D * x + D * ob; }
};

// The online-softmax step of softmax_tile on a 64-key sub-tile (no sink prefix in
// it): visible columns lo .. hi relative to the sub-tile's first key.  P is
// written over the first 32 columns of the sub-tile's S (packed bf16 pairs).
// A warp none of whose rows sees any key of the sub-tile only writes zeros.  The
// return value says whether O must be rescaled: not when the row had seen no key
// before (its O and sum are still zero), only when a finite reference max grows.
__device__ __forceinline__ bool softmax_sub64(uint32_t s_tmem, int lo, int hi, float sl2, float& m_run,
                                              float& l_run, float& alpha) {
  if (__all_sync(0xffffffffu, hi < 0 || lo > 63)) {
    uint32_t z[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) z[i] = 0u;
    tmem_st32(s_tmem, z);
    alpha = 1.0f;
    return false;
  }
  float s[64];
  {
    uint32_t sr[64];
    tmem_ld32_wait(s_tmem, sr);
    tmem_ld32_wait(s_tmem + 32, sr + 32);
#pragma unroll
    for (int i = 0; i < 64; ++i) s[i] = __uint_as_float(sr[i]);
  }
  if (!__all_sync(0xffffffffu, lo <= 0 && hi >= 63)) {
    // visible columns as two 32-bit words, then one shift-and-select per column (a
    // two-sided compare per column took about twice as long, measured)
    const uint32_t w[2] = {range_bits(max(lo, 0), hi, 0), range_bits(max(lo, 0), hi, 32)};
#pragma unroll
    for (int c = 0; c < 64; ++c) s[c] = (static_cast<int>(w[c >> 5] << (31 - (c & 31))) < 0) ? s[c] : -INFINITY;
  }
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = fmaxf(s[2 * i], s[2 * i + 1]);
#pragma unroll
  for (int c = 16; c < 64; c += 16)
#pragma unroll
    for (int i = 0; i < 8; ++i) mx[i] = max3(mx[i], s[c + 2 * i], s[c + 2 * i + 1]);
  const float m_tile = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
  const float m_new = fmaxf(m_run, m_tile);
  const bool fresh = m_run == -INFINITY;               // no key seen yet: O and l are zero
  const bool need = !fresh && (m_new - m_run) * sl2 > 8.0f;
  const float m_use = (need || fresh) ? m_new : m_run;
  alpha = need ? ex2_approx((m_run - m_new) * sl2) : 1.0f;
  const float neg = (m_use == -INFINITY) ? 0.0f : -m_use * sl2;
  const uint64_t scale2 = f2_pack(sl2, sl2), neg2 = f2_pack(neg, neg);
  uint64_t acc[4] = {0, 0, 0, 0};
  uint32_t pr[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    float x0, x1;
    f2_unpack(f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), scale2, neg2), x0, x1);
    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
    acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
    pr[i] = pack_bf16x2(p0, p1);
  }
  float sum0, sum1, sum2, sum3;
  f2_unpack(f2_add(acc[0], acc[1]), sum0, sum1);
  f2_unpack(f2_add(acc[2], acc[3]), sum2, sum3);
  l_run = l_run * alpha + ((sum0 + sum1) + (sum2 + sum3));
  m_run = m_use;
  tmem_st32(s_tmem, pr);
  return need;
}

template <bool OUT_F32>
__global__ void __launch_bounds__(kStreamThreads, 1)
    swa_prefill_stream_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ CUtensorMap tq,
                              const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                              const __grid_constant__ CUtensorMap to) {
  using C = StreamCfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8 * i; };
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(gbase + C::OFF_TMEMPTR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_ABORT);
  int* s_cu = reinterpret_cast<int*>(gbase + C::OFF_TABLES);
  int* s_tpre = s_cu + (kMaxSeqSmem + 1);
  const Ctl ctl{abort_flag, &a};

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < C::NQ; ++i) {
      mbar_init(bar(C::B_QFULL + i), 1);
      mbar_init(bar(C::B_QEMPTY + i), 1);     // the epilogue of the tile that used it
    }
    for (int i = 0; i < C::NKV; ++i) {
      mbar_init(bar(C::B_KVFULL + i), 1);
      mbar_init(bar(C::B_KVEMPTY + i), 2);    // two users, or one user and a stand-in arrive
    }
    for (int i = 0; i < 4; ++i) {          // per warpgroup and S half / O buffer
      mbar_init(bar(C::B_SFULL + i), 1);
      mbar_init(bar(C::B_PFULL + i), 128);
      mbar_init(bar(C::B_OFINAL + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::B_PVDONE + i), 1);
      mbar_init(bar(C::B_DRAIN + i), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kStreamLoadWarp && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    if (!OUT_F32) tma_prefetch_desc(&to);
  }
  if (a.cu_seqlens != nullptr && warp == 0) build_varlen_tables(a, s_cu, s_tpre, lane);
  if (warp == kStreamMmaWarp) {
    tmem_alloc(smem_u32(tmem_ptr), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int total_tiles = a.cu_seqlens != nullptr ? s_tpre[a.n_seq] : a.total_tiles;
  const uint32_t tmem = *tmem_ptr;

  // This CTA's range of query tiles, numbered gq = head * total_tiles + tile (the
  // host keeps Hq * tiles within int32).  Consecutive range tiles li-1, li belong to
  // the same sequence and head exactly when li's tile index qt within its sequence
  // is not 0; then li-1 is tile qt-1 and has already loaded key tile qt-1.  So every
  // range tile loads one new key tile (its diagonal one), except the first tile of
  // the range, which also loads the tile before it when it has one (qt > 0 and a
  // window wider than one key); the ring counter of tile li's diagonal key tile is
  // li + extra.
  const int n_q = a.Hq * total_tiles;
  const int r_lo = static_cast<int>(static_cast<long long>(blockIdx.x) * n_q / gridDim.x);
  const int n_range = static_cast<int>((static_cast<long long>(blockIdx.x) + 1) * n_q / gridDim.x) - r_lo;
  const int tps = (a.L + kBM - 1) / kBM;          // tiles per sequence (fixed-length batches)
  // Unit of range tile li, its head, and the number of query tiles of its sequence.
  auto qtile = [&](int li, Unit& x, int& h, int& seq_tiles) {
    const int gq = r_lo + li;
    h = gq / total_tiles;
    decode_tile(a, s_cu, s_tpre, gq - h * total_tiles, x);
    seq_tiles = a.cu_seqlens != nullptr ? s_tpre[x.seq + 1] - s_tpre[x.seq] : tps;
  };
  int extra = 0;
  if (n_range > 0) {
    Unit x0;
    int h0, st0;
    qtile(0, x0, h0, st0);
    extra = (x0.m0 > 0 && a.window > 1) ? 1 : 0;
  }

  if (warp >= 8) {
  regs_dec<kStreamProducerRegs>();
  if (warp == kStreamLoadWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = (a.debug_flags & 1) == 0;
      int ld = 0;
      int last_fill[C::NKV], last_q[C::NQ];
      for (int i = 0; i < C::NKV; ++i) last_fill[i] = -1;
      for (int i = 0; i < C::NQ; ++i) last_q[i] = -1;
      for (int li = 0; ok && li < n_range; ++li) {
        Unit x;
        int h, seq_tiles;
        qtile(li, x, h, seq_tiles);
        const int kvh = h / a.G;
        const int qs = li % C::NQ;
        if (!(ok = wait_bar(bar(C::B_QEMPTY + qs), ((li / C::NQ) & 1) ^ 1, ctl))) break;
        mbar_expect_tx(bar(C::B_QFULL + qs), C::TILE);
        tma_load_3d(base + C::OFF_Q + qs * C::TILE, &tq, bar(C::B_QFULL + qs), 0, h, x.seq_start + x.m0);
        last_q[qs] = li;
        const int first = (li > 0 && x.m0 > 0) ? x.m1 / kBN : x.kb_lo;
        for (int kt = first; kt <= x.m1 / kBN; ++kt, ++ld) {
          const int st = ld % C::NKV;
          if (!(ok = wait_bar(bar(C::B_KVEMPTY + st), ((ld / C::NKV) & 1) ^ 1, ctl))) break;
          mbar_expect_tx(bar(C::B_KVFULL + st), 2 * C::TILE);
          const uint32_t dst = base + C::OFF_KV + st * 2 * C::TILE;
          tma_load_3d(dst, &tk, bar(C::B_KVFULL + st), 0, kvh, x.seq_start + kt * kBN);
          tma_load_3d(dst + C::TILE, &tv, bar(C::B_KVFULL + st), 0, kvh, x.seq_start + kt * kBN);
          last_fill[st] = ld;
        }
      }
      if (*abort_flag) {
        // Let copies already in flight land before the CTA exits.
        for (int st = 0; st < C::NKV; ++st)
          if (last_fill[st] >= 0) wait_bar(bar(C::B_KVFULL + st), (last_fill[st] / C::NKV) & 1, ctl, false);
        for (int qs = 0; qs < C::NQ; ++qs)
          if (last_q[qs] >= 0) wait_bar(bar(C::B_QFULL + qs), (last_q[qs] / C::NQ) & 1, ctl, false);
      }
    }
    __syncwarp();
  } else if (warp == kStreamMmaWarp || warp == kStreamMmaWarp + 1) {
    // ------------------------------------------------------------ MMA issuers
    const int x = warp - kStreamMmaWarp;             // the softmax warpgroup this thread serves
    if (lane == 0 && x < n_range) {
      bool ok = true;
      const uint32_t s_t = tmem + C::tmem_s(x);
      // one descriptor per operand array, stepped by offsets (slot, sub-tile, k-step)
      const uint64_t dq0 = kmajor_desc<C::QK_STEPS>(base + C::OFF_Q, kBM, 0);
      const uint64_t dk0 = kmajor_desc<C::QK_STEPS>(base + C::OFF_KV, C::SUB, 0);
      const uint64_t dv0 = v_desc<false, C::KSTEP>(base + C::OFF_KV + C::TILE, 0);
      // this warpgroup's 64-key sub-tiles in order: query tiles li = x, x+2, ...,
      // within each the sub-tiles f64 .. l64 of its band
      struct Sub {
        int li, k;                   // range tile, its index among this warpgroup's tiles
        int s64, f64, l64;           // current, first and last sub-tile of the tile
        int m, last_kc;              // diagonal key tile and its ring counter
        bool single_prev, single_diag;
      };
      auto start_tile = [&](Sub& u, int li, int k) -> bool {
        u.li = li;
        u.k = k;
        if (li >= n_range) return false;
        Unit t;
        int h, seq_tiles;
        qtile(li, t, h, seq_tiles);
        const int qt = t.m0 / kBM;
        u.f64 = max(0, t.m0 - a.window + 1) / C::SUB;
        u.l64 = t.m1 / C::SUB;
        u.s64 = u.f64;
        u.m = t.m1 / kBN;
        u.last_kc = li + extra;
        u.single_prev = !(li > 0 && qt > 0);
        u.single_diag = !(li + 1 < n_range && qt + 1 < seq_tiles && a.window > 1);
        return true;
      };
      auto advance = [&](const Sub& u, Sub& v) -> bool {
        v = u;
        if (u.s64 < u.l64) {
          v.s64 = u.s64 + 1;
          return true;
        }
        return start_tile(v, u.li + 2, u.k + 1);
      };
      auto kc_of = [&](const Sub& u) { return u.last_kc - (u.m - (u.s64 >> 1)); };
      // S of sub-tile u = Q K_u^T into half `half` of this warpgroup's S region
      auto issue_qk = [&](const Sub& u, int half) -> bool {
        const int kc = kc_of(u);
        if (u.s64 == u.f64 && !wait_bar(bar(C::B_QFULL + u.li % C::NQ), (u.li / C::NQ) & 1, ctl)) return false;
        if (!wait_bar(bar(C::B_KVFULL + kc % C::NKV), (kc / C::NKV) & 1, ctl)) return false;
        tc_fence_after();
        const uint64_t dq = desc_add(dq0, (u.li % C::NQ) * C::TILE);
        const uint64_t dk = desc_add(dk0, (kc % C::NKV) * 2 * C::TILE + (u.s64 & 1) * (C::SUB * 128));
#pragma unroll
        for (int kk = 0; kk < C::QK_STEPS; ++kk)
          umma_ss<false>(s_t + C::SUB * half, desc_add(dq, kmajor_off<C::QK_STEPS, kBM>(kk)),
                         desc_add(dk, kmajor_off<C::QK_STEPS, C::SUB>(kk)), C::IDESC_QK, kk > 0 ? 1u : 0u);
        tc_commit(bar(C::B_SFULL + 2 * x + half));
        return true;
      };
      Sub cur;
      if (start_tile(cur, x, 0)) {
        ok = issue_qk(cur, 0);
        for (int g = 0; ok; ++g) {
          // one sub-tile ahead: the next S goes into the other half, whose P the
          // previous P V (issued last round, executed in order) has consumed
          Sub nxt;
          const bool more = advance(cur, nxt);
          if (more && !(ok = issue_qk(nxt, (g + 1) & 1))) break;
          if (!(ok = wait_bar(bar(C::B_PFULL + 2 * x + (g & 1)), (g >> 1) & 1, ctl))) break;
          tc_fence_after();
          const int kc = kc_of(cur);
          const uint64_t dv = desc_add(dv0, (kc % C::NKV) * 2 * C::TILE + (cur.s64 & 1) * (C::SUB * 128));
          const uint32_t o_t = tmem + C::tmem_o(x, cur.k & 1);
#pragma unroll
          for (int kk = 0; kk < C::PV_STEPS; ++kk)
            umma_ts<false>(o_t, s_t + C::SUB * (g & 1) + kk * 8, desc_add(dv, mnmajor_off<C::KSTEP>(kk)),
                           C::IDESC_PV, (cur.s64 == cur.f64 && kk == 0) ? 0u : 1u);
          tc_commit(bar(C::B_PVDONE + x));
          if ((cur.s64 & 1) || cur.s64 == cur.l64) {     // this tile's last use of the key tile
            tc_commit(bar(C::B_KVEMPTY + kc % C::NKV));
            if ((cur.s64 >> 1) == cur.m ? cur.single_diag : cur.single_prev)
              mbar_arrive(bar(C::B_KVEMPTY + kc % C::NKV));
          }
          if (cur.s64 == cur.l64) tc_commit(bar(C::B_OFINAL + 2 * x + (cur.k & 1)));
          if (!more) break;
          cur = nxt;
        }
      }
      if (*abort_flag) {
        // Every MMA this thread issued must finish before TMEM is freed.
        tc_commit(bar(C::B_DRAIN + x));
        wait_bar(bar(C::B_DRAIN + x), 0, ctl, false);
      }
    }
    __syncwarp();
  }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    regs_inc<kStreamSoftmaxRegs>();
    const int x_wg = warp >> 2;                      // 0: even range tiles, 1: odd
    const int r = tid & 127;                         // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_tmem = tmem + C::tmem_s(x_wg) + lane_off;
    bool ok = true;
    // the previous query tile of this warpgroup, written out one step late
    bool have_prev = false;
    Unit px{};
    int ph = 0, pli = 0, pk = 0;
    float pm = 0.f, pl = 0.f;
    auto epilogue = [&]() -> bool {
      const int ob = pk & 1;
      if (!__all_sync(0xffffffffu, wait_bar(bar(C::B_OFINAL + 2 * x_wg + ob), (pk >> 1) & 1, ctl))) return false;
      tc_fence_after();
      const uint32_t o_tmem = tmem + C::tmem_o(x_wg, ob) + lane_off;
      const int t = px.m0 + r;
      const int qs = pli % C::NQ;
      if (!OUT_F32 && px.m1 - px.m0 == kBM - 1) {
        // Every MMA that read this Q tile finished before its O was final.
        const uint32_t tile = base + C::OFF_Q + qs * C::TILE;
        stage_row_bf16_d64(o_tmem, gbase + (tile - base), r, a, px, ph, t, pm, pl);
        fence_proxy_async_smem();
        named_bar_sync(1 + x_wg, 128);
        if (r == 0) {
          tma_store_3d(&to, tile, 0, ph, px.seq_start + px.m0);
          bulk_commit();
          bulk_wait_read();
          mbar_arrive(bar(C::B_QEMPTY + qs));
        }
      } else {
        store_row<D, OUT_F32>(o_tmem, a, px, ph, t, pm, pl);
        if (r == 0) mbar_arrive(bar(C::B_QEMPTY + qs));
      }
      return true;
    };
    int g = 0;                                       // this warpgroup's sub-tiles so far
    for (int li = x_wg, k = 0; ok && li < n_range; li += 2, ++k) {
      Unit x;
      int h, seq_tiles;
      qtile(li, x, h, seq_tiles);
      const int t = x.m0 + r;
      const uint32_t o_tmem = tmem + C::tmem_o(x_wg, k & 1) + lane_off;
      const int f64 = max(0, x.m0 - a.window + 1) / C::SUB, l64 = x.m1 / C::SUB;
      float m_run = -INFINITY, l_run = 0.f;
      for (int s64 = f64; s64 <= l64; ++s64, ++g) {
        const int half = g & 1;
        ok = __all_sync(0xffffffffu, wait_bar(bar(C::B_SFULL + 2 * x_wg + half), (g >> 1) & 1, ctl));
        if (!ok) break;
        tc_fence_after();
        float alpha;
        const int n0 = s64 * C::SUB;
        const bool need = softmax_sub64(s_tmem + C::SUB * half, t - a.window + 1 - n0, t - n0, a.scale_log2,
                                        m_run, l_run, alpha);
        if (s64 > f64 && __any_sync(0xffffffffu, need)) {
          // O holds the products of the earlier sub-tiles: wait for the last one
          // (S of this sub-tile being ready implies the one before it has finished)
          ok = __all_sync(0xffffffffu, wait_bar(bar(C::B_PVDONE + x_wg), (g - 1) & 1, ctl));
          if (!ok) break;
          tc_fence_after();
          rescale_o<D>(o_tmem, alpha);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::B_PFULL + 2 * x_wg + half));
        if (s64 == f64 && have_prev) {
          // the previous tile's epilogue, while the tensor pipe works on this one
          if (!(ok = epilogue())) break;
          have_prev = false;
        }
      }
      if (!ok) break;
      have_prev = true;
      px = x;
      ph = h;
      pli = li;
      pk = k;
      pm = m_run;
      pl = l_run;
    }
    if (ok && have_prev) epilogue();
    if (!OUT_F32 && r == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kStreamMmaWarp) tmem_dealloc(tmem, 512);
}

template <bool OUT_F32>
cudaError_t launch_stream_impl(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const CUtensorMap& to, int grid, cudaStream_t stream) {
  static_assert(StreamCfg::SMEM_BYTES <= 232448, "shared memory budget");
  auto kern = swa_prefill_stream_kernel<OUT_F32>;
  // The register split assumes exactly kStreamLaunchRegs per thread at launch; refuse
  // anything else (the caller falls back to the pair kernel).
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kStreamLaunchRegs) return cudaErrorNotSupported;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, StreamCfg::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<grid, kStreamThreads, StreamCfg::SMEM_BYTES, stream>>>(a, tq, tk, tv, to);
  return cudaGetLastError();
}

}  // namespace

bool prefill_stream_supported(int d, bool f32, int window, int n_sink) {
  return d == 64 && !f32 && n_sink == 0 && window >= 1 && window <= kBN + 1;
}

cudaError_t launch_prefill_stream(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const CUtensorMap& to, bool out_f32, int grid,
                                  cudaStream_t stream) {
  return out_f32 ? launch_stream_impl<true>(a, tq, tk, tv, to, grid, stream)
                 : launch_stream_impl<false>(a, tq, tk, tv, to, grid, stream);
}

}  // namespace swa
