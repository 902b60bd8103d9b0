// Eviction composed with the latent cache: slot bookkeeping of a sink + window
// retention budget (close reading §四.10, Table 9 and Appendix J).  Slots
// [0, sink) hold the first history positions; later positions cycle through the
// window slots, each overwriting the position that left the window.  Only
// indices move; the latents of a new token are written by lla_encode into the
// slot computed here, and the decode kernels read slots [0, ctx_len) unchanged.
#include "lla_internal.cuh"

namespace lla {

namespace {

__global__ void evict_append_kernel(int B, int n_cap, int sink, int window,
                                    const int32_t* __restrict__ pos, int64_t* __restrict__ slot,
                                    int32_t* __restrict__ positions, int32_t* __restrict__ ctx_len) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int p = pos[b];
  if (p < 0) {
    slot[b] = -1;
    return;
  }
  const int s = p < sink ? p : sink + (p - sink) % window;
  slot[b] = (int64_t)b * n_cap + s;
  positions[(size_t)b * n_cap + s] = p;
  ctx_len[b] = p + 1 < sink + window ? p + 1 : sink + window;
}

}  // namespace

int64_t evict_slot(int32_t sink, int32_t window, int64_t pos) {
  if (sink < 0 || window < 1 || pos < 0) return -1;
  return pos < sink ? pos : sink + (pos - sink) % window;
}

cudaError_t launch_evict_append(int B, int n_cap, int sink, int window, const int32_t* pos,
                                int64_t* slot, int32_t* positions, int32_t* ctx_len,
                                cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  evict_append_kernel<<<(B + 127) / 128, 128, 0, s>>>(B, n_cap, sink, window, pos, slot, positions,
                                                      ctx_len);
  return cudaGetLastError();
}

}  // namespace lla
