// Launchers of the Based linear branch (Taylor-kernel linear attention),
// dk = 16, dv = 64; fp32 state [B, H, F, dv] and normaliser [B, H, F].
#pragma once
#include <cuda_runtime.h>

namespace swa {

struct BasedLinearArgs {
  const void* q;            // [B, L, H, 16] bf16
  const void* k;            // [B, L, H, 16] bf16
  const void* v;            // [B, L, H, 64] bf16
  void* out;                // [B, L, H, 64] bf16 or fp32
  float* state;             // [B, H, F, 64] or null
  float* zsum;              // [B, H, F] or null (null exactly when state is)
  int B, L, H;
  float scale;
  int out_f32;
  unsigned long long timeout_ns;
  int debug_flags;          // bit 0: the MMA warp issues nothing (the waits then time out);
                            // bit 3: run the CUDA-core chunked kernel instead
  int* err;                 // device status word (first error wins)
};

int based_linear_features(int dk);
cudaError_t launch_based_linear_fwd(const BasedLinearArgs& a, cudaStream_t stream);
cudaError_t launch_based_linear_fwd_simt(const BasedLinearArgs& a, cudaStream_t stream);
cudaError_t launch_based_linear_decode(const void* q, const void* k, const void* v, float* state, float* zsum,
                                       void* out, int B, int H, float scale, bool out_f32, cudaStream_t stream);

}  // namespace swa
