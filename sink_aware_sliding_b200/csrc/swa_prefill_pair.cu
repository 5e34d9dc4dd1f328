// Prefill, two query tiles per CTA (query heads 2p and 2p+1 of the same 128
// rows), sm_100a.
//
// Work unit = (sequence, 128-row query tile, head pair).  Both tiles visit the
// same key tiles (the band plus the sink prefix, nothing else); when the two
// heads read the same KV head (grouped-query attention with an even group) the
// K and V tiles are loaded once for both.  A sink prefix of at most 16 keys left
// of the band is a 16-key mini-tile (sink_mini): its products and softmax cover
// 16 keys instead of a masked 128-key tile.
//
// Roles (384 threads):
//   warps 0-3   softmax of tile A (thread r = query row r = TMEM lane r)
//   warps 4-7   softmax of tile B
//   warp 8      TMA: the two Q tiles of a unit, then the K and V tiles, K one key
//               tile ahead of V, each into the next slot of one ring of tile-sized slots
//   warp 9      tcgen05.mma issue (one thread) and TMEM allocation
// The MMA order per key tile j is
//   O_A += P_A(j) V(j);  S_A = Q_A K(j+1)^T;  O_B += P_B(j) V(j);  S_B = Q_B K(j+1)^T
// so the tensor pipe works on one tile's products while the softmax warps of the
// other tile run, and the two tiles' softmax phases stay half a period apart (with
// one issuer per tile they fell into step and shared the MUFU, 20% slower on a
// B200).  Each tile has a single S region in TMEM (P overwrites S in
// place); because the MMAs of one CTA execute in issue order, S_X(j+1) being
// ready implies O_X += P_X(j) V(j) has finished, so a softmax warp may rescale
// its O rows right after reading S without a further barrier.
// TMEM columns: S_A 0-127, S_B 128-255, O_A 256.., O_B 256+D.. (512 allocated).
// With d = 64 and bf16 output, a unit's finished Q tiles double as the staging
// tiles of its output: each softmax warpgroup writes its normalised O rows there
// in the swizzled layout and one thread stores the tile with TMA; the Q buffer is
// handed back to the load warp only after both stores have read it.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "prefill_common.cuh"

namespace swa {
namespace {

using namespace prefill;

constexpr int kPairThreads = 384;
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
// Register split: launched at 168 per thread (65536 / 384 rounded down to 8) =
// 64512 in all; the load/MMA warpgroup gives back 168 - 88 = 80 per thread
// (10240) and the two softmax warpgroups take 208 - 168 = 40 per thread (10240):
// 2 * 128 * 208 + 128 * 88 = 64512.  The host checks the launch count first.
constexpr int kLaunchRegs = 168;
constexpr uint32_t kSoftmaxRegs = 208;
constexpr uint32_t kProducerRegs = 88;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kProducerRegs == kPairThreads * kLaunchRegs,
              "register split must use exactly the registers the block is launched with");

template <int D, bool F32>
struct PairCfg {
  static constexpr int ELEM = F32 ? 4 : 2;
  static constexpr int CHUNK = 128 / ELEM;          // elements per 128-byte swizzled row
  static constexpr int NCHUNK = D / CHUNK;
  static constexpr int KSTEP = 32 / ELEM;           // K of one MMA instruction (32 bytes)
  static constexpr int QK_STEPS = D / KSTEP;
  static constexpr int PV_STEPS = kBN / KSTEP;
  static constexpr int TILE = kBM * D * ELEM;       // bytes of one Q, K or V tile
  static constexpr int QBUF = TILE <= 16384 ? 2 : 1;     // Q pairs in flight across units
  static constexpr int NSTAGE = TILE <= 16384 ? 8 : 4;   // ring slots, each one K or V tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = OFF_Q + QBUF * 2 * TILE;
  static constexpr int OFF_BAR = OFF_RING + NSTAGE * TILE;
  // barrier indices
  static constexpr int B_QFULL = 0, B_QEMPTY = QBUF, B_FULL = 2 * QBUF, B_EMPTY = B_FULL + NSTAGE,
                       B_SFULL = B_EMPTY + NSTAGE, B_PFULL = B_SFULL + 2, B_OFINAL = B_PFULL + 2,
                       B_DRAIN = B_OFINAL + 2, NBAR = B_DRAIN + 1;
  static constexpr int OFF_TMEMPTR = OFF_BAR + 8 * NBAR;
  static constexpr int OFF_ABORT = OFF_TMEMPTR + 4;
  static constexpr int OFF_TABLES = OFF_ABORT + 12;
  static constexpr int SMEM_BYTES = OFF_TABLES + 2 * 4 * (kMaxSeqSmem + 1) + 1024;
  static constexpr uint32_t IDESC_QK = make_idesc(F32 ? 2u : 1u, kBM, kBN, false);
  static constexpr uint32_t IDESC_QK_SINK = make_idesc(1u, kBM, kSinkMini, false);   // bf16 only
  static constexpr uint32_t IDESC_PV = make_idesc(F32 ? 2u : 1u, kBM, D, true);
  static constexpr bool TMA_STORE = !F32 && D == 64;   // requires QBUF == 2 (see above)
  __device__ static constexpr uint32_t tmem_s(int half) { return half ? 128u : 0u; }
  __device__ static constexpr uint32_t tmem_o(int half) { return 256u + (half ? D : 0); }
};

template <int D, bool F32, bool OUT_F32>
__global__ void __launch_bounds__(kPairThreads, 1)
    swa_prefill_pair_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ CUtensorMap tq,
                            const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                            const __grid_constant__ CUtensorMap to) {
  using C = PairCfg<D, F32>;
  constexpr bool kTmaStore = C::TMA_STORE && !OUT_F32;
  static_assert(!kTmaStore || C::QBUF == 2, "output staging reuses the previous unit's Q buffer");
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
    for (int i = 0; i < C::QBUF; ++i) {
      mbar_init(bar(C::B_QFULL + i), 1);
      // freed by the MMA warp (tcgen05.commit), or by both epilogues after their stores
      mbar_init(bar(C::B_QEMPTY + i), kTmaStore ? 2 : 1);
    }
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(bar(C::B_FULL + i), 1);
      mbar_init(bar(C::B_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::B_SFULL + i), 1);
      mbar_init(bar(C::B_PFULL + i), 128);
      mbar_init(bar(C::B_OFINAL + i), 1);
    }
    mbar_init(bar(C::B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    if (kTmaStore) tma_prefetch_desc(&to);
  }
  if (a.cu_seqlens != nullptr && warp == 0) build_varlen_tables(a, s_cu, s_tpre, lane);
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_ptr), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int total_tiles = a.cu_seqlens != nullptr ? s_tpre[a.n_seq] : a.total_tiles;
  const uint32_t tmem = *tmem_ptr;
  const int n_pairs = a.Hq / 2;
  const int n_units = total_tiles * n_pairs;
  // unit u -> (tile, head pair): heaviest (latest) tiles first
  auto unit_of = [&](int u, Unit& x, int& hA) {
    decode_tile(a, s_cu, s_tpre, total_tiles - 1 - u / n_pairs, x);
    hA = 2 * (u % n_pairs);
  };

  if (warp >= 8) {
  // The load/MMA warpgroup hands registers to the softmax warpgroups (all four of
  // its warps execute this; warps 10 and 11 have no further work).
  regs_dec<kProducerRegs>();
  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const bool skip = (a.debug_flags & 1) != 0;
      bool ok = !skip;
      int ld = 0, uc = 0;
      int last_fill[C::NSTAGE];
      int last_q[C::QBUF];
      for (int i = 0; i < C::NSTAGE; ++i) last_fill[i] = -1;
      for (int i = 0; i < C::QBUF; ++i) last_q[i] = -1;
      for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++uc) {
        Unit x;
        int hA;
        unit_of(u, x, hA);
        const int kvA = hA / a.G, kvB = (hA + 1) / a.G;
        const bool shared = kvA == kvB;
        const int qb = uc % C::QBUF;
        if (!(ok = wait_bar(bar(C::B_QEMPTY + qb), ((uc / C::QBUF) & 1) ^ 1, ctl))) break;
        mbar_expect_tx(bar(C::B_QFULL + qb), 2 * C::TILE);
        for (int half = 0; half < 2; ++half)
          for (int c = 0; c < C::NCHUNK; ++c)
            tma_load_3d(base + C::OFF_Q + (qb * 2 + half) * C::TILE + c * (kBM * 128), &tq,
                        bar(C::B_QFULL + qb), c * C::CHUNK, hA + half, x.seq_start + x.m0);
        last_q[qb] = uc;
        // K runs one key tile ahead of V: K(0), then per tile j K(j+1) and V(j), so that
        // the K tile a Q K^T needs next is requested a whole tile earlier than its V.
        // Each group is one slot (the two heads share a KV head) or two (A, then B).
        const int gsz = shared ? 1 : 2;
        for (int step = 0; ok && step < 2 * x.n_tiles; ++step) {
          const bool is_v = step > 0 && (step % 2 == 0 || step == 2 * x.n_tiles - 1);
          const int j = is_v ? (step == 2 * x.n_tiles - 1 ? x.n_tiles - 1 : step / 2 - 1) : (step + 1) / 2;
          const int row = x.seq_start + tile_n0(x, j);
          for (int part = 0; part < gsz; ++part, ++ld) {
            const int st = ld % C::NSTAGE;
            if (!(ok = wait_bar(bar(C::B_EMPTY + st), ((ld / C::NSTAGE) & 1) ^ 1, ctl))) break;
            const int kvh = part ? kvB : kvA;
            mbar_expect_tx(bar(C::B_FULL + st), C::TILE);
            for (int c = 0; c < C::NCHUNK; ++c)
              tma_load_3d(base + C::OFF_RING + st * C::TILE + c * (kBN * 128), is_v ? &tv : &tk,
                          bar(C::B_FULL + st), c * C::CHUNK, kvh, row);
            last_fill[st] = ld;
          }
        }
      }
      if (*abort_flag) {
        // Let copies already in flight land before the CTA exits.
        for (int st = 0; st < C::NSTAGE; ++st)
          if (last_fill[st] >= 0) wait_bar(bar(C::B_FULL + st), (last_fill[st] / C::NSTAGE) & 1, ctl, false);
        for (int qb = 0; qb < C::QBUF; ++qb)
          if (last_q[qb] >= 0) wait_bar(bar(C::B_QFULL + qb), (last_q[qb] / C::QBUF) & 1, ctl, false);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      int ld = 0, uc = 0, cnt = 0;  // ring counter, units, key tiles processed (both halves)
      auto wait_full = [&](int slot_ctr) -> bool {
        return wait_bar(bar(C::B_FULL + slot_ctr % C::NSTAGE), (slot_ctr / C::NSTAGE) & 1, ctl);
      };
      // descriptors of the first Q tile and of ring slot 0; tiles and k-steps are constant offsets
      constexpr int SPC = C::QK_STEPS / C::NCHUNK;
      const uint64_t dq0 = kmajor_desc<SPC>(base + C::OFF_Q, kBM, 0);
      const uint64_t dk0 = kmajor_desc<SPC>(base + C::OFF_RING, kBN, 0);
      const uint64_t dv0 = v_desc<F32, C::KSTEP>(base + C::OFF_RING, 0);
      auto qk = [&](int half, uint64_t dq, int k_ctr, uint32_t idesc) {
        const uint64_t dk = desc_add(dk0, (k_ctr % C::NSTAGE) * C::TILE);
#pragma unroll
        for (int kk = 0; kk < C::QK_STEPS; ++kk)
          umma_ss<F32>(tmem + C::tmem_s(half), desc_add(dq, kmajor_off<SPC, kBM>(kk)),
                       desc_add(dk, kmajor_off<SPC, kBN>(kk)), idesc, kk > 0 ? 1u : 0u);
        tc_commit(bar(C::B_SFULL + half));
      };
      auto pv = [&](int half, int v_ctr, bool first) {
        const uint64_t dv = desc_add(dv0, (v_ctr % C::NSTAGE) * C::TILE);
#pragma unroll
        for (int kk = 0; kk < C::PV_STEPS; ++kk)
          umma_ts<F32>(tmem + C::tmem_o(half), tmem + C::tmem_s(half) + kk * 8, desc_add(dv, mnmajor_off<C::KSTEP>(kk)),
                       C::IDESC_PV, (first && kk == 0) ? 0u : 1u);
      };
      // P V of the sink mini-tile: one K = 16 step (keys 0..15), starting the accumulator
      auto pv_sink = [&](int half, int v_ctr) {
        umma_ts<F32>(tmem + C::tmem_o(half), tmem + C::tmem_s(half), desc_add(dv0, (v_ctr % C::NSTAGE) * C::TILE),
                     C::IDESC_PV, 0u);
      };
      for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++uc) {
        Unit x;
        int hA;
        unit_of(u, x, hA);
        const bool shared = hA / a.G == (hA + 1) / a.G;
        const int per = shared ? 2 : 4;
        const int qb = uc % C::QBUF;
        const uint64_t qA = desc_add(dq0, (qb * 2) * C::TILE), qB = desc_add(qA, C::TILE);
        if (!(ok = wait_bar(bar(C::B_QFULL + qb), (uc / C::QBUF) & 1, ctl))) break;
        // ring positions in the load order K(0), K(1), V(0), K(2), V(1), ..., V(n-1), in groups
        // of g = per / 2 slots (A, then B when the heads read different KV heads)
        const int g = per / 2, nt = x.n_tiles;
        const bool mini = !F32 && sink_mini(x, a.n_sink);     // key tile 0 is the sink mini-tile
        auto kA = [&](int j) { return ld + (j == 0 ? 0 : (2 * j - 1) * g); };
        auto kB = [&](int j) { return kA(j) + (shared ? 0 : 1); };
        auto vA = [&](int j) { return ld + (j == nt - 1 ? 2 * nt - 1 : 2 * j + 2) * g; };
        auto vB = [&](int j) { return vA(j) + (shared ? 0 : 1); };
        // prologue: S_A(0), S_B(0)
        if (!(ok = wait_full(kA(0)) && (shared || wait_full(kB(0))))) break;
        tc_fence_after();
        // S(0): Q K^T over the first 16 keys only when key tile 0 is the sink mini-tile
        qk(0, qA, kA(0), mini ? C::IDESC_QK_SINK : C::IDESC_QK);
        qk(1, qB, kB(0), mini ? C::IDESC_QK_SINK : C::IDESC_QK);
        tc_commit(bar(C::B_EMPTY + kA(0) % C::NSTAGE));
        if (!shared) tc_commit(bar(C::B_EMPTY + kB(0) % C::NSTAGE));
        if (!kTmaStore && x.n_tiles == 1) tc_commit(bar(C::B_QEMPTY + qb));
        int j0 = 0;
        if (mini) {
          // key tile 0 = the sink mini-tile (a mini unit has band tiles after it, so tile 0
          // is never the last): the same steps as the loop below, with the short P V
          if (!(ok = wait_bar(bar(C::B_PFULL + 0), cnt & 1, ctl) && wait_full(vA(0)))) break;
          tc_fence_after();
          pv_sink(0, vA(0));
          if (!(ok = wait_full(kA(1)) && (shared || wait_full(kB(1))))) break;
          tc_fence_after();
          qk(0, qA, kA(1), C::IDESC_QK);
          if (!(ok = wait_bar(bar(C::B_PFULL + 1), cnt & 1, ctl) && (shared || wait_full(vB(0))))) break;
          tc_fence_after();
          pv_sink(1, vB(0));
          tc_commit(bar(C::B_EMPTY + vA(0) % C::NSTAGE));
          if (!shared) tc_commit(bar(C::B_EMPTY + vB(0) % C::NSTAGE));
          qk(1, qB, kB(1), C::IDESC_QK);
          tc_commit(bar(C::B_EMPTY + kA(1) % C::NSTAGE));
          if (!shared) tc_commit(bar(C::B_EMPTY + kB(1) % C::NSTAGE));
          if (!kTmaStore && x.n_tiles == 2) tc_commit(bar(C::B_QEMPTY + qb));
          j0 = 1;
          ++cnt;
        }
        for (int j = j0; j < x.n_tiles; ++j, ++cnt) {
          const bool last = j == x.n_tiles - 1;
          // The data tiles first: they were requested a tile or more ahead and are in by
          // now, and checking them while P_A is still being written keeps those checks
          // (about 200 cycles each, measured) off the P -> MMA path.
          if (!(ok = wait_full(vA(j)) && (shared || wait_full(vB(j))))) break;
          if (!last && !(ok = wait_full(kA(j + 1)) && (shared || wait_full(kB(j + 1))))) break;
          // ---- tile A: O_A += P_A(j) V(j), then S_A(j+1)
          if (!(ok = wait_bar(bar(C::B_PFULL + 0), cnt & 1, ctl))) break;
          tc_fence_after();
          pv(0, vA(j), j == 0);
          if (last) tc_commit(bar(C::B_OFINAL + 0));
          if (!last) qk(0, qA, kA(j + 1), C::IDESC_QK);
          // ---- tile B: O_B += P_B(j) V(j), then S_B(j+1)
          if (!(ok = wait_bar(bar(C::B_PFULL + 1), cnt & 1, ctl))) break;
          tc_fence_after();
          pv(1, vB(j), j == 0);
          tc_commit(bar(C::B_EMPTY + vA(j) % C::NSTAGE));
          if (!shared) tc_commit(bar(C::B_EMPTY + vB(j) % C::NSTAGE));
          if (last) {
            tc_commit(bar(C::B_OFINAL + 1));
          } else {
            qk(1, qB, kB(j + 1), C::IDESC_QK);
            tc_commit(bar(C::B_EMPTY + kA(j + 1) % C::NSTAGE));
            if (!shared) tc_commit(bar(C::B_EMPTY + kB(j + 1) % C::NSTAGE));
            if (!kTmaStore && j + 1 == x.n_tiles - 1) tc_commit(bar(C::B_QEMPTY + qb));
          }
        }
        ld += x.n_tiles * per;
      }
      if (*abort_flag) {
        // Every MMA this thread issued must finish before TMEM is freed.
        tc_commit(bar(C::B_DRAIN));
        wait_bar(bar(C::B_DRAIN), 0, ctl, false);
      }
    }
    __syncwarp();
  }
  } else {
    // ------------------------------------------------------------ softmax warps
    regs_inc<kSoftmaxRegs>();
    const int half = warp >> 2;                      // 0: tile A, 1: tile B
    const int r = tid & 127;                         // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_tmem = tmem + C::tmem_s(half) + lane_off;
    const uint32_t o_tmem = tmem + C::tmem_o(half) + lane_off;
    int cnt = 0, done_units = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
      const int qb = done_units % C::QBUF;
      Unit x;
      int hA;
      unit_of(u, x, hA);
      const int t = x.m0 + r;
      float m_run = -INFINITY, l_run = 0.f;
      int j0 = 0;
      if (!F32 && sink_mini(x, a.n_sink)) {
        // key tile 0 = the sink mini-tile: the first tile of the unit, so O needs no rescale
        ok = __all_sync(0xffffffffu, wait_bar(bar(C::B_SFULL + half), cnt & 1, ctl));
        if (!ok) break;
        tc_fence_after();
        float alpha;
        softmax_sink16(s_tmem, a.n_sink, a.scale_log2, m_run, l_run, alpha);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::B_PFULL + half));
        j0 = 1;
        ++cnt;
      }
      for (int j = j0; j < x.n_tiles; ++j, ++cnt) {
        ok = __all_sync(0xffffffffu, wait_bar(bar(C::B_SFULL + half), cnt & 1, ctl));
        if (!ok) break;
        tc_fence_after();
        float alpha;
        const bool need = softmax_tile<F32>(s_tmem, x, j, t, a, m_run, l_run, alpha);
        // O_X += P_X(j-1) V(j-1) has finished (it was issued before S_X(j)).
        if (j > 0 && __any_sync(0xffffffffu, need)) rescale_o<D>(o_tmem, alpha);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::B_PFULL + half));
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, wait_bar(bar(C::B_OFINAL + half), done_units & 1, ctl));
      if (!ok) break;
      ++done_units;
      tc_fence_after();
      if constexpr (kTmaStore) {
        // Every MMA that read this unit's Q tiles finished before O_X was final.
        const uint32_t tile = base + C::OFF_Q + (qb * 2 + half) * C::TILE;
        if (x.m1 - x.m0 == kBM - 1) {
          stage_row_bf16_d64(o_tmem, gbase + (tile - base), r, a, x, hA + half, t, m_run, l_run);
          fence_proxy_async_smem();
          named_bar_sync(1 + half, 128);
          if (r == 0) {
            tma_store_3d(&to, tile, 0, hA + half, x.seq_start + x.m0);
            bulk_commit();
            bulk_wait_read();
            mbar_arrive(bar(C::B_QEMPTY + qb));
          }
        } else {
          store_row<D, OUT_F32>(o_tmem, a, x, hA + half, t, m_run, l_run);
          named_bar_sync(1 + half, 128);
          if (r == 0) mbar_arrive(bar(C::B_QEMPTY + qb));
        }
      } else {
        store_row<D, OUT_F32>(o_tmem, a, x, hA + half, t, m_run, l_run);
      }
    }
    if (kTmaStore && r == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

template <int D, bool F32, bool OUT_F32>
cudaError_t launch_pair_impl(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, const CUtensorMap& to, int grid, cudaStream_t stream) {
  using C = PairCfg<D, F32>;
  static_assert(C::SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(OUT_F32 || !F32, "fp32 inputs give fp32 outputs");
  auto kern = swa_prefill_pair_kernel<D, F32, OUT_F32>;
  // The register split inside the kernel assumes exactly kLaunchRegs per thread at launch;
  // anything else could leave setmaxnreg.inc waiting, so refuse (the caller falls back).
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorNotSupported;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<grid, kPairThreads, C::SMEM_BYTES, stream>>>(a, tq, tk, tv, to);
  return cudaGetLastError();
}

}  // namespace

bool prefill_pair_supported(int Hq, int G, int d, bool f32) {
  if (Hq % 2 != 0) return false;
  const int tile = 128 * d * (f32 ? 4 : 2);
  // The ring must hold two key tiles' slots: 2 slots per tile when the heads share
  // a KV head, 4 otherwise (only the 8-slot ring of 16 KB tiles fits that).
  return G % 2 == 0 || tile <= 16384;
}

cudaError_t launch_prefill_pair(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, const CUtensorMap& to, int d, bool f32,
                                bool out_f32, int grid, cudaStream_t stream) {
  if (f32) {
    if (d == 64) return launch_pair_impl<64, true, true>(a, tq, tk, tv, to, grid, stream);
    return cudaErrorInvalidValue;
  }
  if (out_f32) {
    if (d == 64) return launch_pair_impl<64, false, true>(a, tq, tk, tv, to, grid, stream);
    if (d == 128) return launch_pair_impl<128, false, true>(a, tq, tk, tv, to, grid, stream);
    return cudaErrorInvalidValue;
  }
  if (d == 64) return launch_pair_impl<64, false, false>(a, tq, tk, tv, to, grid, stream);
  if (d == 128) return launch_pair_impl<128, false, false>(a, tq, tk, tv, to, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace swa
