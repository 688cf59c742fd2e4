// append.cu - mla_cache_append kernel: scatter new tokens' latent and rotated key into
// the paged cache, one warp per token (append.cuh).
#include "append.cuh"

namespace mla {

__global__ void __launch_bounds__(256) cache_append_kernel(AppendParams p) {
  grid_dep_wait();
  grid_dep_launch();
  const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= int64_t(p.batch) * p.n_new) return;
  append_token(p, gw, lane);
}

cudaError_t launch_cache_append(const AppendParams& p, cudaStream_t stream) {
  const int64_t ntok = int64_t(p.batch) * p.n_new;
  if (ntok == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (ntok * 32 + threads - 1) / threads;
  return launch_pdl(cache_append_kernel, dim3(unsigned(blocks)), dim3(threads), 0, stream, 1, p);
}

}  // namespace mla
