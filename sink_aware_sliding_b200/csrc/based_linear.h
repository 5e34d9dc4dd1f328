// Launchers of the Based linear branch (Taylor-kernel linear attention),
// dk = 16, dv = 64; fp32 state [B, H, F, dv] and normaliser [B, H, F].
#pragma once
#include <cuda_runtime.h>

namespace swa {

int based_linear_features(int dk);
cudaError_t launch_based_linear_fwd(const void* q, const void* k, const void* v, void* out, float* state,
                                    float* zsum, int B, int L, int H, float scale, bool out_f32,
                                    cudaStream_t stream);
cudaError_t launch_based_linear_decode(const void* q, const void* k, const void* v, float* state, float* zsum,
                                       void* out, int B, int H, float scale, bool out_f32, cudaStream_t stream);

}  // namespace swa
