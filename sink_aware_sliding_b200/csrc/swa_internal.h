// Internal launch interfaces shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace swa {

constexpr int kBM = 128;            // query rows per prefill tile (TMEM lanes)
constexpr int kBN = 128;            // keys per prefill tile
constexpr int kMaxSeqSmem = 1024;   // varlen sequences whose tables fit in shared memory

struct PrefillArgs {
  void* out;
  float* lse;                 // may be null
  const int32_t* cu_seqlens;  // null: n_seq sequences of length L laid end to end
  int n_seq;
  int L;
  long long T;                // total tokens
  int Hq, Hkv, G;
  int window, n_sink;
  float scale;
  float scale_log2;           // scale * log2(e)
  int lse_varlen;             // 1: lse [Hq, T]; 0: lse [n_seq, Hq, L]
  int total_tiles;            // fixed length: n_seq * ceil(L / kBM); varlen: computed on device
  unsigned long long timeout_ns;
  int debug_flags;
  int* err;
};

// Launch the persistent prefill kernel (d = 64 or 128; bf16 in with bf16 or fp32 out, or
// fp32 in and out with d = 64).
cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tv, int d, bool f32, bool out_f32, int grid,
                           cudaStream_t stream);

// Two-query-tile prefill (heads 2p, 2p+1 per CTA); used when Hq is even and the
// ring can hold two key tiles (always for 16 KB tiles, else when pairs share a KV head).
// Backward pass: dq [n_seq, L, Hq, d], dk/dv [n_seq, L, Hkv, d] (fp32, written, not
// accumulated) from q, k, v, the forward's out and lse and dout (bf16).
struct BwdArgs {
  PrefillArgs pa;       // geometry: n_seq sequences of length L, heads, window, sinks, scale
  const void* out;      // [n_seq, L, Hq, d] bf16
  const void* dout;     // [n_seq, L, Hq, d] bf16
  const float* lse;     // [n_seq, Hq, L]
  float* dq;
  float* dk;
  float* dv;
};
cudaError_t launch_bwd(const BwdArgs& ba, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, int d, cudaStream_t stream);

// Short-window stream kernel: d = 64, bf16 inputs, window <= 129, no sink prefix.
bool prefill_stream_supported(int d, bool f32, int window, int n_sink);
cudaError_t launch_prefill_stream(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const CUtensorMap& to, bool out_f32, int grid,
                                  cudaStream_t stream);
bool prefill_pair_supported(int Hq, int G, int d, bool f32);
// `to` maps the output (bf16, same box as q); it is used for d = 64 bf16 output only.
cudaError_t launch_prefill_pair(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, const CUtensorMap& to, int d, bool f32,
                                bool out_f32, int grid, cudaStream_t stream);

struct DecodeArgs {
  const void* q;        // [B, Hq, d]
  const void* kcache;   // [B, Hkv, W, d]
  const void* vcache;
  const void* sink_k;   // [B, Hkv, S, d]
  const void* sink_v;
  const int32_t* pos;   // [B]
  void* out;            // [B, Hq, d], bf16 or (out_f32) float32
  float* lse;           // [B, Hq] or null
  float* part;          // partial states, (n_warps + B*Hkv) slots
  int B, Hq, Hkv, G, W, S;
  float scale_log2;
  int n_warps;          // total warps of the split kernel
  int out_f32;          // 1: out is float32
};

// Rotary frequencies theta_i = base^(-2i/d), i < d/2 (d <= 128), for the fused
// rotary encoding.
struct RopeTable {
  double theta[64];
};
void make_rope_table(double base, int d, RopeTable* t);

// rope == nullptr: q is used as given; otherwise q is rotated at pos[b] first.
cudaError_t launch_decode(const DecodeArgs& a, int d, int grid, int block, cudaStream_t stream,
                          const RopeTable* rope = nullptr);
size_t decode_partial_floats(int G, int d);
// Every argument check of swa_decode_ex except the workspace (SWA_OK when the
// arguments are valid; B == 0 is valid and means nothing to launch).
int decode_args_status(const void* q, const void* kcache, const void* vcache, const void* sink_k,
                       const void* sink_v, const int32_t* pos, const void* out, const float* lse, int B,
                       int Hq, int Hkv, int d, int window, int n_sink, float scale, int out_dtype);
cudaError_t decode_occupancy(int d, int B, int* ctas_per_sm);
int decode_threads();

cudaError_t launch_cache_fill(const void* k, const void* v, int P, void* kc, void* vc, void* sk,
                              void* sv, int B, int Hkv, int d, int W, int S, cudaStream_t stream);
cudaError_t launch_cache_append(const void* k, const void* v, const int32_t* pos, void* kc,
                                void* vc, void* sk, void* sv, int B, int Hkv, int d, int W, int S,
                                cudaStream_t stream);

// Rotary encoding in place: q [T, Hq, d], k [T, Hkv, d] (k may be null), token t
// at positions[t]; and the fused rotate-k-then-append of one decode step.
cudaError_t launch_rope_qk(void* q, void* k, const int32_t* positions, long long T, int Hq, int Hkv,
                           int d, const RopeTable& rt, cudaStream_t stream);
cudaError_t launch_rope_append(const void* k, const void* v, const int32_t* pos, void* kc, void* vc,
                               void* sk, void* sv, int B, int Hkv, int d, int W, int S,
                               const RopeTable& rt, cudaStream_t stream);

// One hybrid decode step: the window branch (append, decode; d = 64) and the Based
// linear branch (recurrent step; dk = 16, dv = 64) in one launch.
struct HybridArgs {
  const void* q;            // [B, Hq, 64] bf16
  const void* k_new;        // [B, Hkv, 64] bf16
  const void* v_new;
  const int32_t* pos;       // [B]
  void* kcache;             // [B, Hkv, W, 64] bf16
  void* vcache;
  void* sink_k;             // [B, Hkv, S, 64] bf16 (unused when S == 0)
  void* sink_v;
  void* out;                // [B, Hq, 64] bf16
  float* lse;               // [B, Hq] or null
  int B, Hq, Hkv, G, W, S;
  float scale_log2;
  const void* ql;           // [B, H_l, 16] bf16
  const void* kl;
  const void* vl;           // [B, H_l, 64] bf16
  float* state;             // [B, H_l, 273, 64]
  float* zsum;              // [B, H_l, 273]
  void* out_l;              // [B, H_l, 64] bf16
  int H_l;
  float scale_l;
};
bool hybrid_window_supported(int d, int window, int n_sink);
cudaError_t launch_hybrid_decode(const HybridArgs& a, cudaStream_t stream);

// Hadamard output projection z = alpha * (y H) + beta over rows of n = 2^k elements.
struct HadamardArgs {
  const void* y;            // [n_rows, n] bf16
  const float* alpha;       // [n]
  const float* beta;        // [n]
  void* z;                  // [n_rows, n] bf16 or f32
  long long n_rows;
  unsigned long long timeout_ns;
  int debug_flags;          // bit 0: issue no loads (the waits then time out)
  int* err;                 // device status word (first error wins)
};
cudaError_t launch_hadamard(const HadamardArgs& a, int n, bool out_f32, int sms, cudaStream_t stream);

}  // namespace swa
