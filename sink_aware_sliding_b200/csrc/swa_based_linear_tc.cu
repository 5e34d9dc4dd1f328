// Prefill of the Based linear branch on the tensor cores (tcgen05, bf16
// operands, fp32 accumulators in tensor memory).  The method is the second-order
// Taylor linear attention described in swa_based_linear.cu ("Simple linear
// attention language models balance the recall-throughput tradeoff", proposed
// method): out_t = phi(q_t) S_t / phi(q_t).z_t with S_t = sum_{s<=t} phi(k_s) v_s^T.
//
// The quadratic part of phi(q).phi(k) = 1 + x + x^2/2 is symmetric in the pair
// (a, b), so the kernel uses the 136 products with a <= b instead of all 256:
// u_a^2 with weight scale/sqrt(2) and u_a u_b (a < b) with weight scale, whose
// dot products give the same kernel.  Internal feature order: the 16 linear
// terms sqrt(scale) u, the constant 1, the 136 products (a-major), zeros up to
// 192 columns; 153 are real.  The state is returned in the interface order
// [1, linear, all 256 products], an off-diagonal internal row split back as
// row / sqrt(2) into (a, b) and (b, a).
//
// One CTA per (sequence, head) walks the sequence in chunks of 128 tokens.  With
// V1 = [V | 1 | 0...] (the values, a column of ones that turns the same products
// into the normaliser, zero padding) a chunk is
//   X   = phi_lin(Q) phi_lin(K)^T                  (= scale q.k; K = 16)
//   O   = phi(Q) S_bf16 + kappa_causal(X) V1        (S from the earlier chunks)
//   S^T += V1^T phi(K)                              (M = value column, N = 192 features)
// with kappa(x) = 1 + x + x^2/2 under the causal mask and out = O[:, :64] / O[:, 64].
// S is accumulated transposed (tensor-memory lane = value column), so that each
// lane's row is one row of the K-major bf16 operand of the next chunk's phi(Q) S.
// phi(Q) and phi(K) have buffers of their own and V1 and O two each, so the
// feature rows of the next chunk are written while this chunk's products run.
//
// Roles (416 threads):
//   warps 0-3   token rows of the K side: k loads, phi(K), kappa(X) -> P (bf16,
//               over X's own tensor-memory columns);
//   warps 4-7   token rows of the Q side and state lanes: q and v loads, phi(Q),
//               V1, S^T -> S_bf16 between chunks, the final state;
//   warps 8-11  part of S^T -> S_bf16, the output epilogue out = O[:, :64] / O[:, 64];
//   warp 12     one thread issues every MMA, per chunk in the order phi(Q) S, X,
//               the state update, P V1 (so that the state update never waits for P).
// All waits on mbarriers are bounded; on a time-out the CTA stops, drains its
// MMAs, frees its tensor memory and records the status.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <utility>

#include "based_linear.h"
#include "ptx.cuh"

namespace swa {
namespace {

namespace bl {
constexpr int kChunk = 128;                  // tokens per chunk (MMA M)
constexpr int kDK = 16, kDV = 64;
constexpr int kF = 1 + kDK + kDK * kDK;      // 273 features in the interface order
constexpr int kFI = 192;                     // internal feature columns (153 real)
constexpr int kFReal = kDK + 1 + kDK * (kDK + 1) / 2;   // 153
constexpr int kNV = 80;                      // V1 columns: 64 values, the ones column, padding
constexpr int kQSteps = 10;                  // phi(Q) S_bf16 over features 0 .. 159 (K steps of 16)
constexpr int kGranules = 20;                // 16-byte granules of a feature row written per chunk (0 .. 159)
constexpr int kThreads = 416;
constexpr int kMmaWarp = 12;
constexpr uint32_t kCh = kChunk * 128;       // one 64-column chunk of a 128-row operand: 16 KB
constexpr uint32_t kSbCh = kNV * 128;        // one 64-column chunk of S_bf16 (80 rows): 10 KB
constexpr uint32_t OFF_PHIQ = 0;             // [128 tokens x 192 features], 3 chunks
constexpr uint32_t OFF_PHIK = 3 * kCh;
constexpr uint32_t OFF_V1 = 6 * kCh;         // two buffers of [values chunk | ones chunk]
constexpr uint32_t OFF_SB = 10 * kCh;        // S_bf16 [80 value columns x 192 features], 3 chunks
constexpr uint32_t OFF_QST = OFF_SB + 3 * kSbCh;   // q rows of two chunks (32 bytes a row)
constexpr uint32_t OFF_KST = OFF_QST + 2 * kChunk * 32;  // k rows of two chunks
constexpr uint32_t OFF_BAR = OFF_KST + 2 * kChunk * 32;
enum {
  B_PHIQ, B_PHIK, B_V1, B_V1b, B_X, B_O1, B_P, B_OFULL, B_OFULLb, B_OFREE, B_OFREEb, B_SFULL, B_SB, B_DRAIN,
  kNumBars
};
constexpr uint32_t OFF_TMEMPTR = OFF_BAR + kNumBars * 8;
constexpr uint32_t OFF_ABORT = OFF_TMEMPTR + 4;
constexpr uint32_t kSmemUsed = OFF_ABORT + 4;
constexpr uint32_t kSmem = kSmemUsed + 1024;  // slack to align the base to 1024 bytes
static_assert(kSmem <= 232448, "shared memory");
// tensor-memory columns
constexpr uint32_t T_X = 0;                  // X (fp32, 128 columns); P (bf16 pairs) over its first 64
constexpr uint32_t T_O = 128;                // O buffer j at T_O + 80 j (80 columns each)
constexpr uint32_t T_ST = 288;               // S^T: lanes = value columns, 192 feature columns
// instruction descriptors (bf16 x bf16 -> fp32); bit 15 makes A MN-major
constexpr uint32_t IDESC_X = make_idesc(1, 128, 128, false);
constexpr uint32_t IDESC_QS = make_idesc(1, 128, kNV, false);
constexpr uint32_t IDESC_PV = make_idesc(1, 128, kNV, true);
constexpr uint32_t IDESC_KV = make_idesc(1, 128, kFI, true) | (1u << 15);
constexpr int kStatusTimeout = 4;            // SWA_ERR_DEVICE_TIMEOUT

// Product p (0 .. 135) of the symmetric pairs a <= b in a-major order.
__host__ __device__ constexpr int pair_a(int p) {
  int a = 0;
  while (p >= kDK - a) {
    p -= kDK - a;
    ++a;
  }
  return a;
}
__host__ __device__ constexpr int pair_b(int p) {
  int a = 0;
  while (p >= kDK - a) {
    p -= kDK - a;
    ++a;
  }
  return a + p;
}
}  // namespace bl

// K-major operand with 128-byte rows in 64-column chunks of `chunk` bytes: K step kk (16 columns).
__device__ __forceinline__ uint64_t bl_kdesc(uint32_t base, uint32_t chunk, int kk) {
  return smem_desc(base + (kk >> 2) * chunk + (kk & 3) * 32, 16, 1024, kLayoutSw128);
}
// MN-major operand (rows = K, 64-element chunks along M or N, `chunk` bytes apart): K step kk (16 rows).
__device__ __forceinline__ uint64_t bl_mndesc(uint32_t base, uint32_t chunk, int kk) {
  return smem_desc(base + kk * 16 * 128, chunk, 1024, kLayoutSw128);
}
// 16-byte granule g of row r in a 128-byte-swizzled chunk.
__device__ __forceinline__ uint32_t gran(uint32_t chunk_base, int r, int g) {
  return chunk_base + r * 128 + (((g ^ r) & 7) << 4);
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t a) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}
// 64 or 96 consecutive columns of this warp's 32 lanes, then one wait::ld (one asm block,
// so that no register is read before the data has arrived).
__device__ __forceinline__ void ld64_wait(uint32_t t, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]),"=r"(r[1]),"=r"(r[2]),"=r"(r[3]),"=r"(r[4]),"=r"(r[5]),"=r"(r[6]),"=r"(r[7]),"=r"(r[8]),"=r"(r[9]),"=r"(r[10]),"=r"(r[11]),"=r"(r[12]),"=r"(r[13]),"=r"(r[14]),"=r"(r[15]),"=r"(r[16]),"=r"(r[17]),"=r"(r[18]),"=r"(r[19]),"=r"(r[20]),"=r"(r[21]),"=r"(r[22]),"=r"(r[23]),"=r"(r[24]),"=r"(r[25]),"=r"(r[26]),"=r"(r[27]),"=r"(r[28]),"=r"(r[29]),"=r"(r[30]),"=r"(r[31]),
        "=r"(r[32]),"=r"(r[33]),"=r"(r[34]),"=r"(r[35]),"=r"(r[36]),"=r"(r[37]),"=r"(r[38]),"=r"(r[39]),"=r"(r[40]),"=r"(r[41]),"=r"(r[42]),"=r"(r[43]),"=r"(r[44]),"=r"(r[45]),"=r"(r[46]),"=r"(r[47]),"=r"(r[48]),"=r"(r[49]),"=r"(r[50]),"=r"(r[51]),"=r"(r[52]),"=r"(r[53]),"=r"(r[54]),"=r"(r[55]),"=r"(r[56]),"=r"(r[57]),"=r"(r[58]),"=r"(r[59]),"=r"(r[60]),"=r"(r[61]),"=r"(r[62]),"=r"(r[63])
      : "r"(t), "r"(t + 32)
      : "memory");
}
__device__ __forceinline__ void ld96_wait(uint32_t t, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%96];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%97];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95}, [%98];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]),"=r"(r[1]),"=r"(r[2]),"=r"(r[3]),"=r"(r[4]),"=r"(r[5]),"=r"(r[6]),"=r"(r[7]),"=r"(r[8]),"=r"(r[9]),"=r"(r[10]),"=r"(r[11]),"=r"(r[12]),"=r"(r[13]),"=r"(r[14]),"=r"(r[15]),"=r"(r[16]),"=r"(r[17]),"=r"(r[18]),"=r"(r[19]),"=r"(r[20]),"=r"(r[21]),"=r"(r[22]),"=r"(r[23]),"=r"(r[24]),"=r"(r[25]),"=r"(r[26]),"=r"(r[27]),"=r"(r[28]),"=r"(r[29]),"=r"(r[30]),"=r"(r[31]),
        "=r"(r[32]),"=r"(r[33]),"=r"(r[34]),"=r"(r[35]),"=r"(r[36]),"=r"(r[37]),"=r"(r[38]),"=r"(r[39]),"=r"(r[40]),"=r"(r[41]),"=r"(r[42]),"=r"(r[43]),"=r"(r[44]),"=r"(r[45]),"=r"(r[46]),"=r"(r[47]),"=r"(r[48]),"=r"(r[49]),"=r"(r[50]),"=r"(r[51]),"=r"(r[52]),"=r"(r[53]),"=r"(r[54]),"=r"(r[55]),"=r"(r[56]),"=r"(r[57]),"=r"(r[58]),"=r"(r[59]),"=r"(r[60]),"=r"(r[61]),"=r"(r[62]),"=r"(r[63]),
        "=r"(r[64]),"=r"(r[65]),"=r"(r[66]),"=r"(r[67]),"=r"(r[68]),"=r"(r[69]),"=r"(r[70]),"=r"(r[71]),"=r"(r[72]),"=r"(r[73]),"=r"(r[74]),"=r"(r[75]),"=r"(r[76]),"=r"(r[77]),"=r"(r[78]),"=r"(r[79]),"=r"(r[80]),"=r"(r[81]),"=r"(r[82]),"=r"(r[83]),"=r"(r[84]),"=r"(r[85]),"=r"(r[86]),"=r"(r[87]),"=r"(r[88]),"=r"(r[89]),"=r"(r[90]),"=r"(r[91]),"=r"(r[92]),"=r"(r[93]),"=r"(r[94]),"=r"(r[95])
      : "r"(t), "r"(t + 32), "r"(t + 64)
      : "memory");
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// 16-byte asynchronous copy global -> shared (zero-filled when src_bytes = 0); the
// copies are tracked by commit groups, not by the thread's registers, so a later
// barrier wait does not wait for them.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

struct BlCtl {
  volatile int* abort_flag;
  const BasedLinearArgs* a;
};
// Bounded wait; false on time-out (which starts the CTA's abort) or once another
// thread has started it (unless honor_abort is false, as in the teardown).
__device__ __forceinline__ bool bl_wait(uint32_t bar, uint32_t parity, const BlCtl& c, bool honor_abort = true) {
  for (int i = 0; i < 128; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (honor_abort && *c.abort_flag) return false;
    if (globaltimer_ns() - t0 > c.a->timeout_ns) {
      *c.abort_flag = 1;
      atomicCAS(c.a->err, 0, bl::kStatusTimeout);
      return false;
    }
  }
}
// The same wait taken by a whole warp: true only if every lane's wait succeeded, so
// that the warp-collective tensor-memory accesses that follow run converged.
__device__ __forceinline__ bool bl_warp_wait(uint32_t bar, uint32_t parity, const BlCtl& c) {
  const bool ok = bl_wait(bar, parity, c);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void unpack16(const uint4& lo, const uint4& hi, float* u) {
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    u[2 * i] = bf_lo(w[i]);
    u[2 * i + 1] = bf_hi(w[i]);
  }
}

// The vectors a feature row is formed from: u, sqrt(scale) u, scale u and
// scale/sqrt(2) u, and the constant feature (0 for a row past the sequence's end,
// whose u is zero as well).
struct FeatIn {
  float u[bl::kDK], ru[bl::kDK], su[bl::kDK], cu[bl::kDK];
  float one;
};
// Internal feature F (compile-time).
template <int F>
__device__ __forceinline__ float feat(const FeatIn& x) {
  using namespace bl;
  if constexpr (F < kDK) {
    return x.ru[F];
  } else if constexpr (F == kDK) {
    return x.one;
  } else if constexpr (F < kFReal) {
    constexpr int a = pair_a(F - kDK - 1), b = pair_b(F - kDK - 1);
    return (a == b ? x.cu[a] : x.su[a]) * x.u[b];
  } else {
    return 0.0f;
  }
}
template <int G>
__device__ __forceinline__ void write_granule(uint32_t phi, int t, const FeatIn& x) {
  constexpr int f = 8 * G;
  sts128(gran(phi + (G >> 3) * bl::kCh, t, G & 7), pack_bf16x2(feat<f>(x), feat<f + 1>(x)),
         pack_bf16x2(feat<f + 2>(x), feat<f + 3>(x)), pack_bf16x2(feat<f + 4>(x), feat<f + 5>(x)),
         pack_bf16x2(feat<f + 6>(x), feat<f + 7>(x)));
}
template <int... G>
__device__ __forceinline__ void write_granules(uint32_t phi, int t, const FeatIn& x, std::integer_sequence<int, G...>) {
  (write_granule<G>(phi, t, x), ...);
}
// Row t of phi(u) (internal order, features 0 .. 159) into a K-major feature operand
// from the bf16 row (two 16-byte words); keep = false writes a zero row.
__device__ __forceinline__ void write_phi_row(uint32_t phi, int t, const uint4& lo, const uint4& hi, float rs,
                                              float c2, float s, bool keep) {
  FeatIn x;
  unpack16(lo, hi, x.u);
#pragma unroll
  for (int e = 0; e < bl::kDK; ++e) {
    x.u[e] = keep ? x.u[e] : 0.f;
    x.ru[e] = rs * x.u[e];
    x.su[e] = s * x.u[e];
    x.cu[e] = c2 * x.u[e];
  }
  x.one = keep ? 1.0f : 0.0f;
  write_granules(phi, t, x, std::make_integer_sequence<int, bl::kGranules>{});
}

// Internal feature F of one state lane (value column n < 64, or z for n = 64) into the
// interface layout [1, linear (16), products (256, row-major)].
template <int F>
__device__ __forceinline__ void store_state_feature(float val, int n, float* st, float* zs) {
  using namespace bl;
  if constexpr (F < kFReal) {
    auto put = [&](int fa, float x) {
      if (n < kDV) st[fa * kDV + n] = x;
      else zs[fa] = x;
    };
    if constexpr (F < kDK) {
      put(1 + F, val);
    } else if constexpr (F == kDK) {
      put(0, val);
    } else {
      constexpr int a = pair_a(F - kDK - 1), b = pair_b(F - kDK - 1);
      if constexpr (a == b) {
        put(1 + kDK + kDK * a + a, val);
      } else {
        const float h = val * 0.70710678118654752f;
        put(1 + kDK + kDK * a + b, h);
        put(1 + kDK + kDK * b + a, h);
      }
    }
  }
}
template <int P, int... E>
__device__ __forceinline__ void store_state_piece(const uint32_t* sr, int n, float* st, float* zs,
                                                  std::integer_sequence<int, E...>) {
  (store_state_feature<32 * P + E>(__uint_as_float(sr[E]), n, st, zs), ...);
}

// S^T columns 32 p0 .. 32 p1 - 1 (features) of this warp's lanes -> rows of S_bf16
// (lane n = value column; lanes 80 and up hold nothing).  Warp-collective.
__device__ __forceinline__ void convert_state(uint32_t tmem_lane, uint32_t sb, int n, int p0, int p1) {
#pragma unroll 1
  for (int p = p0; p < p1; ++p) {
    uint32_t sr[32];
    tmem_ld32_wait(tmem_lane + bl::T_ST + 32 * p, sr);
    if (n < bl::kNV) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int G = 4 * p + g;
        sts128(gran(sb + (G >> 3) * bl::kSbCh, n, G & 7),
               pack_bf16x2(__uint_as_float(sr[8 * g]), __uint_as_float(sr[8 * g + 1])),
               pack_bf16x2(__uint_as_float(sr[8 * g + 2]), __uint_as_float(sr[8 * g + 3])),
               pack_bf16x2(__uint_as_float(sr[8 * g + 4]), __uint_as_float(sr[8 * g + 5])),
               pack_bf16x2(__uint_as_float(sr[8 * g + 6]), __uint_as_float(sr[8 * g + 7])));
      }
    }
  }
}

// 13 warps: one of the four SM sub-partitions holds four of them, and its 16K
// registers cap every thread at 128 (ptxas applies the cap from these bounds).
__global__ void __launch_bounds__(bl::kThreads, 1)
    swa_based_linear_tc_kernel(const __grid_constant__ BasedLinearArgs a) {
  using namespace bl;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + OFF_BAR + 8u * i; };
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(gbase + OFF_TMEMPTR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + OFF_ABORT);
  const BlCtl ctl{abort_flag, &a};

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int nc = (a.L + kChunk - 1) / kChunk;

  // zero both feature operands (their padding columns stay zero), S_bf16 and the
  // ones chunks of both V1 buffers, then put the ones in place (column 64 = 1.0)
  for (uint32_t o = tid * 16; o < 6 * kCh; o += kThreads * 16) sts128(base + OFF_PHIQ + o, 0, 0, 0, 0);
  for (uint32_t o = tid * 16; o < 3 * kSbCh; o += kThreads * 16) sts128(base + OFF_SB + o, 0, 0, 0, 0);
  for (uint32_t o = tid * 16; o < kCh; o += kThreads * 16) {
    sts128(base + OFF_V1 + kCh + o, 0, 0, 0, 0);
    sts128(base + OFF_V1 + 3 * kCh + o, 0, 0, 0, 0);
  }
  __syncthreads();
  if (tid < kChunk) {
    sts32(gran(base + OFF_V1 + kCh, tid, 0), 0x3F80u);
    sts32(gran(base + OFF_V1 + 3 * kCh, tid, 0), 0x3F80u);
  }
  fence_proxy_async_smem();
  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const bool threads = i == B_PHIQ || i == B_PHIK || i == B_V1 || i == B_V1b || i == B_P || i == B_OFREE ||
                           i == B_OFREEb;
      mbar_init(bar(i), i == B_SB ? 256 : (threads ? 128 : 1));
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_ptr), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const float sc = a.scale, c2 = a.scale * 0.70710678118654752f, rs = sqrtf(a.scale);

  if (warp < 4) {
    // ---------------------------------------------------------------- K-side token rows
    const int t = tid;                                   // row of the chunk = tensor-memory lane
    const uint32_t lane_t = static_cast<uint32_t>(warp * 32) << 16;
    const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(a.k);
    // k row t of chunk c -> staging buffer c & 1 (a commit group of its own)
    auto copy_k = [&](int c) {
      const int tok = c * kChunk + t;
      const bool in = c < nc && tok < a.L;
      const __nv_bfloat16* src = in ? kg + ((static_cast<long long>(b) * a.L + tok) * a.H + h) * kDK : kg;
      const uint32_t dst = base + OFF_KST + (c & 1) * kChunk * 32 + t * 32;
      cp_async16(dst, src, in ? 16u : 0u);
      cp_async16(dst + 16, src + 8, in ? 16u : 0u);
      cp_async_commit();
    };
    copy_k(0);
    copy_k(1);
    bool ok = true;
    for (int i = 0; i < nc && ok; ++i) {
      const int n = min(kChunk, a.L - i * kChunk);
      // phi(K) once the previous chunk's products are done with the operand
      if (i > 0 && !(ok = bl_warp_wait(bar(B_SFULL), (i - 1) & 1, ctl))) break;
      cp_async_wait<1>();                                // k of chunk i (chunk i+1's may be in flight)
      {
        const uint32_t src = base + OFF_KST + (i & 1) * kChunk * 32 + t * 32;
        write_phi_row(base + OFF_PHIK, t, lds128(src), lds128(src + 16), rs, c2, sc, t < n);
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(B_PHIK));
      copy_k(i + 2);                                     // into the buffer just read
      // kappa(X) with the causal mask -> P (bf16 pairs over X's first 64 columns)
      if (!(ok = bl_warp_wait(bar(B_X), i & 1, ctl))) break;
      tc_fence_after();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t xr[64], pr[32];
        ld64_wait(tmem + lane_t + T_X + 64 * half, xr);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int s0 = 64 * half + 2 * j;
          const float x0 = __uint_as_float(xr[2 * j]), x1 = __uint_as_float(xr[2 * j + 1]);
          const float k0 = s0 <= t ? fmaf(x0, fmaf(0.5f, x0, 1.f), 1.f) : 0.f;
          const float k1 = s0 + 1 <= t ? fmaf(x1, fmaf(0.5f, x1, 1.f), 1.f) : 0.f;
          pr[j] = pack_bf16x2(k0, k1);
        }
        tmem_st32(tmem + lane_t + T_X + 32 * half, pr);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_P));
    }
    cp_async_wait<0>();
  } else if (warp < 8) {
    // ---------------------------------------------------------------- Q-side token rows, state lanes
    const int r = tid - 128;                             // token row (phi(Q), V1) and state lane
    const int w = warp - 4;                              // tensor-memory lane quarter
    const uint32_t lane_t = static_cast<uint32_t>(w * 32) << 16;
    const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q);
    const __nv_bfloat16* vg = static_cast<const __nv_bfloat16*>(a.v);
    // Asynchronous copies of chunk c: its v rows into V1 buffer c & 1 (16-byte granules,
    // swizzled as the MMA reads them) and its q rows into staging buffer c & 1.  Each
    // call is one commit group.
    auto copy_v = [&](int c) {
      const int tok = c * kChunk + r;
      const bool in = c < nc && tok < a.L;
      const __nv_bfloat16* src = in ? vg + ((static_cast<long long>(b) * a.L + tok) * a.H + h) * kDV : vg;
      const uint32_t vb = base + OFF_V1 + (c & 1) * 2 * kCh;
#pragma unroll
      for (int g = 0; g < 8; ++g) cp_async16(gran(vb, r, g), src + 8 * g, in ? 16u : 0u);
      cp_async_commit();
    };
    auto copy_q = [&](int c) {
      const int tok = c * kChunk + r;
      const bool in = c < nc && tok < a.L;
      const __nv_bfloat16* src = in ? qg + ((static_cast<long long>(b) * a.L + tok) * a.H + h) * kDK : qg;
      const uint32_t dst = base + OFF_QST + (c & 1) * kChunk * 32 + r * 32;
      cp_async16(dst, src, in ? 16u : 0u);
      cp_async16(dst + 16, src + 8, in ? 16u : 0u);
      cp_async_commit();
    };
    auto v_ready = [&](int c) {                          // after its copies have landed
      fence_proxy_async_smem();
      mbar_arrive(bar(B_V1 + (c & 1)));
    };
    auto put_q = [&](int c) {                            // after its copies have landed
      const uint32_t src = base + OFF_QST + (c & 1) * kChunk * 32 + r * 32;
      write_phi_row(base + OFF_PHIQ, r, lds128(src), lds128(src + 16), rs, c2, sc, true);
      fence_proxy_async_smem();
      mbar_arrive(bar(B_PHIQ));
    };
    bool ok = true;
    if (nc > 0) {
      copy_v(0);
      copy_q(0);
      cp_async_wait<0>();
      v_ready(0);
      put_q(0);
      copy_q(1);
    }
    for (int i = 0; i < nc && ok; ++i) {
      if (i > 0) {
        // S^T after chunk i-1 -> S_bf16 (row n = value column, K-major over the features)
        if (!(ok = bl_warp_wait(bar(B_SFULL), (i - 1) & 1, ctl))) break;
        tc_fence_after();
        // features 0 .. 95 here, 96 .. 159 in the epilogue warps
        if (w < 3) convert_state(tmem + lane_t, base + OFF_SB, 32 * w + lane, 0, 3);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(B_SB));
      }
      // commit groups in flight: at most [v(i)], [q(i+1)] (issued in the previous round)
      if (i > 0) {
        cp_async_wait<1>();                              // v(i) landed
        v_ready(i);
      }
      if (i + 1 < nc) {
        // the other V1 buffer was last read by chunk i-1's state update (done: B_SFULL
        // above) and its P V1, issued after it
        if (i > 0 && !(ok = bl_warp_wait(bar(B_OFULL + ((i - 1) & 1)), ((i - 1) >> 1) & 1, ctl))) break;
        copy_v(i + 1);
        // phi(Q) of chunk i+1 once chunk i's products are done with the operand
        if (!(ok = bl_warp_wait(bar(B_O1), i & 1, ctl))) break;
        cp_async_wait<1>();                              // q(i+1) landed (v(i+1) may be in flight)
        put_q(i + 1);
        copy_q(i + 2);
      }
    }
    cp_async_wait<0>();
    // final state, in the layout [1, linear, products] x (64 values | z)
    if (ok && a.state != nullptr) {
      const long long sb = static_cast<long long>(bh) * kF;
      if (nc == 0) {
        for (int f = r; f < kF; f += 128) {
          float4* dst = reinterpret_cast<float4*>(a.state + (sb + f) * kDV);
#pragma unroll
          for (int c = 0; c < 16; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
          a.zsum[sb + f] = 0.f;
        }
      } else if (bl_warp_wait(bar(B_SFULL), (nc - 1) & 1, ctl)) {
        tc_fence_after();
        if (w < 3) {
          const int n = 32 * w + lane;
          float* st = a.state + sb * kDV;
          float* zs = a.zsum + sb;
          uint32_t sr[32];
#define SWA_BL_STATE_PIECE(P)                                                               \
  tmem_ld32_wait(tmem + lane_t + T_ST + 32 * (P), sr);                                      \
  if (n <= kDV) store_state_piece<P>(sr, n, st, zs, std::make_integer_sequence<int, 32>{});
          SWA_BL_STATE_PIECE(0)
          SWA_BL_STATE_PIECE(1)
          SWA_BL_STATE_PIECE(2)
          SWA_BL_STATE_PIECE(3)
          SWA_BL_STATE_PIECE(4)
#undef SWA_BL_STATE_PIECE
        }
      }
    }
  } else if (warp < 12) {
    // ---------------------------------------------------------------- output epilogue
    const int t = tid - 256;                             // row of the chunk = tensor-memory lane
    const uint32_t lane_t = static_cast<uint32_t>((warp - 8) * 32) << 16;
    for (int i = 0; i < nc; ++i) {
      const int n = min(kChunk, a.L - i * kChunk);
      const int ob = i & 1;
      if (i + 1 < nc) {
        // features 96 .. 159 of S^T after chunk i -> S_bf16 for chunk i+1 (the rest in
        // warps 4-6); the state update of chunk i completes before its P V1
        if (!bl_warp_wait(bar(B_SFULL), i & 1, ctl)) break;
        tc_fence_after();
        if (warp < 11) convert_state(tmem + lane_t, base + OFF_SB, t, 3, 5);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(B_SB));
      }
      if (!bl_warp_wait(bar(B_OFULL + ob), (i >> 1) & 1, ctl)) break;
      tc_fence_after();
      uint32_t orr[96];
      ld96_wait(tmem + lane_t + T_O + 80 * ob, orr);
      tc_fence_before();
      mbar_arrive(bar(B_OFREE + ob));
      if (t < n) {
        const float inv = 1.0f / __uint_as_float(orr[64]);
        const long long row = (static_cast<long long>(b) * a.L + i * kChunk + t) * a.H + h;
        if (a.out_f32) {
          float4* o = reinterpret_cast<float4*>(static_cast<float*>(a.out) + row * kDV);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            o[c] = make_float4(__uint_as_float(orr[4 * c]) * inv, __uint_as_float(orr[4 * c + 1]) * inv,
                               __uint_as_float(orr[4 * c + 2]) * inv, __uint_as_float(orr[4 * c + 3]) * inv);
        } else {
          uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + row * kDV);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t* w = orr + 8 * c;
            o[c] = make_uint4(pack_bf16x2(__uint_as_float(w[0]) * inv, __uint_as_float(w[1]) * inv),
                              pack_bf16x2(__uint_as_float(w[2]) * inv, __uint_as_float(w[3]) * inv),
                              pack_bf16x2(__uint_as_float(w[4]) * inv, __uint_as_float(w[5]) * inv),
                              pack_bf16x2(__uint_as_float(w[6]) * inv, __uint_as_float(w[7]) * inv));
          }
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && (a.debug_flags & 1) == 0) {
      bool ok = true;
      for (int i = 0; i < nc && ok; ++i) {
        const int ob = i & 1;
        if (!(ok = bl_wait(bar(B_PHIQ), i & 1, ctl))) break;
        if (i > 0) {
          // O = phi(Q) S_bf16 needs phi(Q), the converted state and a drained O buffer
          if (!(ok = bl_wait(bar(B_SB), (i - 1) & 1, ctl))) break;
          if (i > 1 && !(ok = bl_wait(bar(B_OFREE + ob), ((i - 2) >> 1) & 1, ctl))) break;
          tc_fence_after();
#pragma unroll 1
          for (int kk = 0; kk < kQSteps; ++kk)
            umma_ss<false>(tmem + T_O + 80 * ob, bl_kdesc(base + OFF_PHIQ, kCh, kk), bl_kdesc(base + OFF_SB, kSbCh, kk),
                           IDESC_QS, kk > 0 ? 1u : 0u);
        }
        if (!(ok = bl_wait(bar(B_PHIK), i & 1, ctl))) break;
        // X overwrites P: chunk i-1's P V1 must be done
        if (i > 0 && !(ok = bl_wait(bar(B_OFULL + (ob ^ 1)), ((i - 1) >> 1) & 1, ctl))) break;
        tc_fence_after();
        // X = phi_lin(Q) phi_lin(K)^T: the first 16 feature columns of both operands
        umma_ss<false>(tmem + T_X, bl_kdesc(base + OFF_PHIQ, kCh, 0), bl_kdesc(base + OFF_PHIK, kCh, 0), IDESC_X, 0u);
        tc_commit(bar(B_X));
        tc_commit(bar(B_O1));
        const uint32_t v1 = base + OFF_V1 + ob * 2 * kCh;
        if (!(ok = bl_wait(bar(B_V1 + ob), (i >> 1) & 1, ctl))) break;
        tc_fence_after();
        // S^T += V1^T phi(K): A = V1 read MN-major (M = value columns), B = phi(K) MN-major (N = features)
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          umma_ss<false>(tmem + T_ST, bl_mndesc(v1, kCh, kk), bl_mndesc(base + OFF_PHIK, kCh, kk), IDESC_KV,
                         (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(B_SFULL));
        if (!(ok = bl_wait(bar(B_P), i & 1, ctl))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          umma_ts<false>(tmem + T_O + 80 * ob, tmem + T_X + kk * 8, bl_mndesc(v1, kCh, kk), IDESC_PV,
                         (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(B_OFULL + ob));
      }
      // let every issued MMA finish before the tensor memory is freed
      tc_commit(bar(B_DRAIN));
      bl_wait(bar(B_DRAIN), 0, ctl, false);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_based_linear_fwd(const BasedLinearArgs& a, cudaStream_t stream) {
  if (a.debug_flags & 8) return launch_based_linear_fwd_simt(a, stream);
  cudaError_t e = cudaFuncSetAttribute(swa_based_linear_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(bl::kSmem));
  if (e != cudaSuccess) return e;
  swa_based_linear_tc_kernel<<<a.B * a.H, bl::kThreads, bl::kSmem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace swa
