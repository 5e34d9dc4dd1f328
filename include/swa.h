/*
 * libswa — causal sliding-window softmax attention with attention sinks on
 * NVIDIA B200 (sm_100a).  C ABI: plain pointers and sizes, no framework types.
 *
 * The operation ("Sliding-window beats linear attention", section 1 Key Terms
 * and section 3): query position t of a sequence attends to the keys
 *     S(t) = { j : j <= t  and  ( j >= t - window + 1  or  j < n_sink ) },
 * i.e. a causal window of `window` keys ending at t plus the first `n_sink`
 * positions of its sequence (the attention sinks), which stay visible at every
 * position; a key that is both is counted once.  With G = Hq / Hkv, query head
 * h reads KV head h / G (grouped-query attention, "Rethinking Attention Output
 * Projection", section 1).  For each (t, h):
 *     z_j = scale * <q_t,h , k_j,kvh>,  out = softmax_j(z) . v,  lse = ln sum_j exp(z_j).
 *
 * Conventions shared by every entry point:
 *   - Every device pointer is owned by the caller, must stay valid until the
 *     work queued on `stream` has finished, and must be 16-byte aligned.
 *     The library allocates no device memory and keeps no device state except
 *     one error word per device (see swa_device_error).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  The return value reports argument errors
 *     (nothing launched) and launch errors only; a device-side wait that ran
 *     past its time limit is reported through swa_device_error.
 *   - The library keeps, per device, addresses it looked up once (its error
 *     word, and swa_decode_noalloc's scratch array).  It must not be used on a
 *     device after cudaDeviceReset, or after its primary context was destroyed
 *     and created again, within the same process.
 *   - bf16 is IEEE bfloat16 stored as uint16; f32 is IEEE binary32.
 *   - Accumulation is fp32.  In the bf16 path the softmax numerators P are
 *     rounded to bf16 (round-to-nearest-even) before the P.V product and the
 *     output is rounded to bf16; the fp32 path runs both products as tf32.
 */
#ifndef SWA_H
#define SWA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* swa_stream_t; /* same type as cudaStream_t */

typedef enum {
  SWA_OK = 0,
  SWA_ERR_INVALID_ARG = 1,    /* a size, pointer or alignment precondition failed; nothing launched */
  SWA_ERR_UNSUPPORTED = 2,    /* valid arguments outside what the kernels implement (e.g. d = 96) */
  SWA_ERR_CUDA = 3,           /* the CUDA runtime or driver reported an error */
  SWA_ERR_DEVICE_TIMEOUT = 4, /* a kernel gave up on a barrier wait (swa_device_error only) */
  SWA_ERR_WORKSPACE = 5       /* workspace pointer missing or smaller than required */
} swa_status;

/* Element types of q, k, v / out. */
typedef enum {
  SWA_DTYPE_BF16 = 0,         /* bf16 in, bf16 out */
  SWA_DTYPE_F32 = 1,          /* f32 in, f32 out (products run as tf32) */
  SWA_DTYPE_BF16_F32OUT = 2   /* bf16 in, f32 out (same arithmetic as SWA_DTYPE_BF16, no final rounding) */
} swa_dtype;

/*
 * Prefill over B sequences of equal length L.
 *   q   [B, L, Hq, d]    input type     (row-major, contiguous)
 *   k,v [B, L, Hkv, d]   input type
 *   out [B, L, Hq, d]    output type    (written)
 *   lse [B, Hq, L]       float32        (written; may be NULL)
 * Requires Hq % Hkv == 0, window >= 1, n_sink >= 0, scale > 0 and finite.
 * Supported: bf16 inputs (either output type) with d in {64, 128}; f32 with d = 64.
 * Nothing is launched (and SWA_OK returned) when B * L == 0.
 */
int swa_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
            int B, int Hq, int Hkv, int L, int d, int window, int n_sink, float scale,
            int dtype, swa_stream_t stream);

/*
 * Prefill over n_seq packed sequences of different lengths; sequence i owns
 * tokens cu_seqlens[i] .. cu_seqlens[i+1]-1 and its window and sinks are
 * counted from its own first token.
 *   q   [T, Hq, d], k,v [T, Hkv, d] (input type), out [T, Hq, d] (output type)
 *   lse [Hq, T]      float32 (may be NULL)
 *   cu_seqlens       DEVICE int32 [n_seq + 1], non-decreasing, cu_seqlens[0] = 0,
 *                    cu_seqlens[n_seq] = T (not checked: the device reads it)
 * Requires 1 <= n_seq <= 1024 and the same head/dtype preconditions as swa_fwd.
 */
int swa_fwd_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                   const int32_t* cu_seqlens, int n_seq, long long T,
                   int Hq, int Hkv, int d, int window, int n_sink, float scale,
                   int dtype, swa_stream_t stream);

/*
 * Ring-buffer KV cache for decoding ("Sliding-window beats linear attention",
 * section 1: sliding-window attention needs a fixed amount of memory at
 * inference; section 3: the sinks must be kept).  Layout, all bf16:
 *   kcache, vcache  [B, Hkv, window, d]   position p lives in slot p mod window
 *   sink_k, sink_v  [B, Hkv, n_sink, d]   position p < n_sink also lives in sink slot p
 * Writing position p overwrites slot p mod window, which evicts position
 * p - window.  Sink slots are written once and never evicted.
 */

/*
 * Fill an empty cache with the prefix positions 0 .. P-1 of k, v [B, P, Hkv, d]
 * (bf16).  Only the last min(P, window) positions reach the ring and only
 * positions < n_sink reach the sink slots.  sink_k/sink_v may be NULL when
 * n_sink == 0.  P == 0 launches nothing.
 */
int swa_cache_fill(const void* k, const void* v, int P,
                   void* kcache, void* vcache, void* sink_k, void* sink_v,
                   int B, int Hkv, int d, int window, int n_sink, swa_stream_t stream);

/*
 * Append one token per sequence: k_new, v_new [B, Hkv, d] (bf16) are written at
 * position pos[b] (DEVICE int32 [B], pos[b] >= 0) into slot pos[b] mod window,
 * and into sink slot pos[b] when pos[b] < n_sink.
 */
int swa_cache_append(const void* k_new, const void* v_new, const int32_t* pos,
                     void* kcache, void* vcache, void* sink_k, void* sink_v,
                     int B, int Hkv, int d, int window, int n_sink, swa_stream_t stream);

/*
 * Bytes of device workspace swa_decode needs for these sizes (fp32 split
 * partials).  Pure host function; 0 means the sizes are invalid.
 */
size_t swa_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int window, int n_sink);

/*
 * One decode step: query q [B, Hq, d] (bf16) of position pos[b] attends to the
 * cached keys of S(pos[b]): ring slots holding positions max(0, pos-window+1)
 * .. pos and the sink slots j < min(n_sink, pos - window + 1).  The caller must
 * have appended position pos[b] (and every earlier one) before this call.
 *   out [B, Hq, d] bf16 (written), lse [B, Hq] float32 (written; may be NULL)
 *   workspace: device buffer of at least swa_decode_workspace_bytes(...) bytes,
 *   256-byte aligned; contents need not be initialised and are scratch.
 * The keys are split evenly over the GPU's warps (split-K); the partial
 * softmax states are merged by their log-sum-exps in a second kernel.
 * Supported: d in {64, 128}, Hq / Hkv <= 8.
 */
int swa_decode(const void* q, const void* kcache, const void* vcache,
               const void* sink_k, const void* sink_v, const int32_t* pos,
               void* out, float* lse,
               int B, int Hq, int Hkv, int d, int window, int n_sink, float scale,
               void* workspace, size_t workspace_bytes, swa_stream_t stream);

/*
 * swa_decode with a choice of output type: out_dtype SWA_DTYPE_BF16 writes out
 * as bf16 (exactly swa_decode), SWA_DTYPE_BF16_F32OUT writes it as float32 (the
 * same arithmetic without the final rounding, for checking the kernels'
 * arithmetic on its own).  Anything else is SWA_ERR_INVALID_ARG.
 */
int swa_decode_ex(const void* q, const void* kcache, const void* vcache,
                  const void* sink_k, const void* sink_v, const int32_t* pos,
                  void* out, float* lse,
                  int B, int Hq, int Hkv, int d, int window, int n_sink, float scale,
                  int out_dtype, void* workspace, size_t workspace_bytes, swa_stream_t stream);

/*
 * swa_decode without a workspace argument, for callers that cannot allocate
 * device memory: code that runs inside a host framework which owns every
 * device allocation (a serving engine with a preallocated arena, a plugin in
 * somebody else's process), or under a rule that forbids cudaMalloc after
 * start-up because allocation can stall the device or fail at the worst time.
 * The pages have no counterpart; this is a packaging variant of swa_decode.
 *
 * Same arguments, layouts and results as swa_decode minus workspace and
 * workspace_bytes.  The scratch for the partial softmax states is a fixed
 * 8 MiB array compiled into the library (every GPU that loads the library
 * holds it until the process exits); nothing is allocated, by the library or
 * any library it calls.  Sizes whose scratch (swa_decode_workspace_bytes)
 * exceeds 8 MiB are rejected with SWA_ERR_UNSUPPORTED and nothing is launched;
 * for the 64 x 32 x 8 x 128 decode workload the need is about 3.5 MiB.
 * The first call on each device looks up that device's address of the array
 * (cudaGetSymbolAddress, with the device current); make that first call
 * before any stream capture.  With CUDA's lazy module loading (the default
 * since CUDA 12.2) the library's device code, this array included, is loaded
 * onto a device when the library is first used there, which can be that first
 * call: a caller that may not allocate after start-up makes one call (any
 * valid decode) at start-up, or sets CUDA_MODULE_LOADING=EAGER.  The argument
 * checks of swa_decode come first (SWA_ERR_INVALID_ARG / SWA_ERR_UNSUPPORTED as
 * there), then the size check against the array.  All calls on a device share the one array and
 * it keeps whatever the last call left there; every value a call reads was
 * written earlier in the same call, so nothing needs clearing, but calls
 * whose work overlaps on the GPU (different streams, or different host
 * threads) race on the array and must be serialised by the caller.
 */
int swa_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                       const void* sink_k, const void* sink_v, const int32_t* pos,
                       void* out, float* lse,
                       int B, int Hq, int Hkv, int d, int window, int n_sink, float scale,
                       swa_stream_t stream);

/*
 * Backward pass of sink-aware sliding-window attention (the gradients of the
 * forward above; visible set of "Sliding-window beats linear attention",
 * sections 1 and 3).  With P the forward's weights (recomputed from lse) and
 * D_t = rowsum(dout_t * out_t):
 *   dv = P^T dout,  dS = P * (dout v^T - D),  dq = scale dS k,  dk = scale dS^T q,
 * the gradients of a KV head summed over the query heads that read it.
 *   q, out, dout [B, L, Hq, d] bf16;  k, v [B, L, Hkv, d] bf16   (read)
 *   lse [B, Hq, L] float32: the forward's log-sum-exp                (read)
 *   dq [B, L, Hq, d], dk, dv [B, L, Hkv, d] float32                   (written)
 * Supported: d = 64 or 128, fixed-length batches.  Arguments and errors as
 * swa_fwd; a bounded device wait that runs out sets SWA_ERR_DEVICE_TIMEOUT.
 */
int swa_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
            float* dq, float* dk, float* dv, int B, int Hq, int Hkv, int L, int d, int window, int n_sink,
            float scale, swa_stream_t stream);

/*
 * Rotary position encoding of the sliding-window branch ("Simple linear
 * attention language models balance the recall-throughput tradeoff", proposed
 * method: the window attention uses rotary position encoding, the linear branch
 * none).  The page gives no formula; reading used: the RoFormer rotation with
 * rotate-half pairs.  For i < d/2 the pair (x[i], x[i + d/2]) of a vector at
 * absolute position p turns by the angle p * theta_i, theta_i =
 * rope_base^(-2i/d) (10000 is the usual base):
 *   x'[i] = x[i] cos - x[i+d/2] sin,   x'[i+d/2] = x[i] sin + x[i+d/2] cos.
 * The angle is formed in double precision and reduced to [-pi, pi] before a
 * single-precision sine/cosine; the rotated values are rounded to bf16 (RNE).
 * A cached key keeps the rotation of its own position; nothing is re-indexed
 * inside the window.  Supported d: 64, 128.  rope_base > 0 and finite.
 *
 * swa_rope_qk: rotates in place q [n_tokens, Hq, d] and k [n_tokens, Hkv, d]
 * (bf16, device, 16-byte aligned; k may be NULL to rotate q alone, or Hq = 0
 * to rotate k alone), token t at positions[t] (int32, device).  Used before
 * swa_fwd / swa_fwd_varlen, whose kernels take rotated q and k.
 */
int swa_rope_qk(void* q, void* k, const int32_t* positions, long long n_tokens, int Hq, int Hkv, int d,
                double rope_base, swa_stream_t stream);

/*
 * swa_cache_append with the new key rotated at pos[b] first (one launch): the
 * decode step's "rotate k on append".  Arguments as swa_cache_append plus
 * rope_base; v_new is stored unchanged.
 */
int swa_rope_cache_append(const void* k_new, const void* v_new, const int32_t* pos, void* kcache,
                          void* vcache, void* sink_k, void* sink_v, int B, int Hkv, int d, int window,
                          int n_sink, double rope_base, swa_stream_t stream);

/*
 * swa_decode with the query rotated at pos[b] inside the decode kernel (the
 * decode step's "rotate q"); the cache must hold rotated keys (swa_rope_qk
 * before swa_cache_fill, swa_rope_cache_append per step).  Arguments, workspace
 * (same size as swa_decode's) and errors as swa_decode, plus rope_base.
 */
int swa_decode_rope(const void* q, const void* kcache, const void* vcache, const void* sink_k,
                    const void* sink_v, const int32_t* pos, void* out, float* lse, int B, int Hq,
                    int Hkv, int d, int window, int n_sink, float scale, double rope_base,
                    void* workspace, size_t workspace_bytes, swa_stream_t stream);

/*
 * The linear-attention branch of the Based hybrid ("Simple linear attention
 * language models balance the recall-throughput tradeoff", proposed method: a
 * linear attention whose feature dimension sets the recurrent state, no
 * position encoding).  The pages give no feature map; reading used: the
 * second-order Taylor kernel of exp, kappa(q, k) = 1 + x + x^2/2 with
 * x = scale q.k, i.e. features phi(u) = [1, sqrt(scale) u, scale vec(u u^T)/sqrt(2)]
 * (F = 1 + dk + dk^2 entries, the outer product row-major), and causal
 * normalisation: out_t = sum_{s<=t} kappa(q_t,k_s) v_s / sum_{s<=t} kappa(q_t,k_s).
 * The recurrent state is S = sum phi(k_s) v_s^T [F, dv] and z = sum phi(k_s) [F].
 * Supported: dk = 16, dv = 64.  Prefill runs on the tensor cores with bf16
 * features, bf16 kernel values kappa within a chunk and a bf16 copy of the
 * state as operands, fp32 accumulation; the state itself is kept in fp32.
 * Decode is fp32 throughout.  Every pointer must be 16-byte aligned
 * (SWA_ERR_INVALID_ARG otherwise); tensors are contiguous.  A device-side wait
 * that runs out sets SWA_ERR_DEVICE_TIMEOUT (read with swa_device_error).
 *
 * swa_based_linear_state_features(dk) = F.
 * swa_based_linear_fwd: q, k [B, L, H, dk], v [B, L, H, dv] bf16 (read);
 *   out [B, L, H, dv] bf16 or float32 (out_dtype SWA_DTYPE_BF16 / SWA_DTYPE_F32);
 *   state [B, H, F, dv] and zsum [B, H, F] float32: both NULL, or both written
 *   with the state after position L-1 (to continue with swa_based_linear_decode).
 * swa_based_linear_decode: one generated token per sequence: q, k [B, H, dk],
 *   v [B, H, dv] bf16; state and zsum are updated in place with the token
 *   (S += phi(k) v^T, z += phi(k)) and out [B, H, dv] = phi(q) S / phi(q).z.
 */
int swa_based_linear_state_features(int dk);
int swa_based_linear_fwd(const void* q, const void* k, const void* v, void* out, float* state, float* zsum,
                         int B, int L, int H, int dk, int dv, float scale, int out_dtype, swa_stream_t stream);
int swa_based_linear_decode(const void* q, const void* k, const void* v, float* state, float* zsum, void* out,
                            int B, int H, int dk, int dv, float scale, int out_dtype, swa_stream_t stream);

/*
 * One generated token of a Based-style hybrid layer ("Simple linear attention
 * language models balance the recall-throughput tradeoff", proposed method: a
 * sliding window and a linear attention side by side) in one launch: the window
 * branch's swa_cache_append + swa_decode and the linear branch's
 * swa_based_linear_decode, with the same results as those calls in sequence.
 *   window branch: q [B, Hq, d], k_new, v_new [B, Hkv, d] bf16 at positions pos
 *     (DEVICE int32 [B]); the ring cache and sink slots as for swa_cache_append
 *     (sink_k/sink_v may be NULL when n_sink == 0); out [B, Hq, d] bf16, lse [B, Hq]
 *     float32 (may be NULL).  Supported: d = 64 and window + n_sink <= 512.
 *   linear branch: ql, kl [B, H_l, dk], vl [B, H_l, dv] bf16; state, zsum updated in
 *     place; out_l [B, H_l, dv] bf16.  Supported: dk = 16, dv = 64.
 * Argument errors return SWA_ERR_INVALID_ARG / SWA_ERR_UNSUPPORTED with nothing
 * launched; every pointer must be 16-byte aligned (pos and lse 4-byte).
 */
int swa_hybrid_decode(const void* q, const void* k_new, const void* v_new, const int32_t* pos,
                      void* kcache, void* vcache, void* sink_k, void* sink_v, void* out, float* lse,
                      int B, int Hq, int Hkv, int d, int window, int n_sink, float scale,
                      const void* ql, const void* kl, const void* vl, float* state, float* zsum,
                      void* out_l, int H_l, int dk, int dv, float scale_l, swa_stream_t stream);

/*
 * Hadamard output projection, the step after attention ("Rethinking Attention
 * Output Projection: Structured Hadamard Transforms for Efficient Transformers",
 * section 2): per row, z = alpha * (y H) + beta, where H is the fixed Walsh-
 * Hadamard matrix, which preserves the l2 norm.  Reading used: H is the
 * Sylvester-ordered matrix of size n normalised by 1/sqrt(n),
 * H[i][j] = (-1)^popcount(i & j) / sqrt(n), computed as a fast Walsh-Hadamard
 * transform; y is a row of attention output with the heads concatenated
 * (n = Hq * d, the [.., Hq, d] layout of swa_fwd / swa_decode outputs).
 *   y     [n_rows, n] bf16              (read)
 *   alpha, beta [n]   float32           (read; the learned rescaling)
 *   z     [n_rows, n] bf16 or float32 per out_dtype (SWA_DTYPE_BF16 / SWA_DTYPE_F32)
 * Supported: n a power of two with 32 <= n <= 8192.  fp32 arithmetic.
 */
int swa_hadamard_proj(const void* y, const float* alpha, const float* beta, void* z,
                      long long n_rows, int n, int out_dtype, swa_stream_t stream);

/* Static text for a status code. */
const char* swa_status_string(int status);

/*
 * Synchronises `stream`, then returns and clears the current device's error
 * word: SWA_OK, or SWA_ERR_DEVICE_TIMEOUT when a kernel abandoned a barrier
 * wait after the time limit (it then wrote no output and released its tensor
 * memory).  Returns SWA_ERR_CUDA if the synchronisation itself failed.
 */
int swa_device_error(swa_stream_t stream);

/* The same call under a second name: reads and clears the device error word. */
int swa_debug_error_word(swa_stream_t stream);

/*
 * Time limit, in nanoseconds, of every device-side barrier wait launched after
 * this call (default 2e9).  Process-wide.  Returns the previous value.
 */
unsigned long long swa_set_wait_timeout_ns(unsigned long long ns);

/*
 * Test hooks, process-wide.  Bit 0 makes the prefill kernels' load warp issue
 * no copies, so that its consumers' bounded waits run out; bit 1 makes
 * swa_fwd / swa_fwd_varlen use the one-query-tile kernel even where another
 * kernel applies; bit 2 keeps them off the short-window stream kernel (d = 64,
 * window <= 129, no sinks), so the two-tile kernel runs instead.  For
 * swa_based_linear_fwd, bit 0 makes the MMA warp issue nothing (the other warps'
 * bounded waits run out) and bit 3 runs the fp32 CUDA-core form of the same
 * chunked step instead of the tensor-core kernel.  0 restores normal operation.
 * Returns the previous flags.
 */
int swa_set_debug_flags(int flags);

/* Library version, e.g. 0x000100 for 0.1.0. */
int swa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SWA_H */
