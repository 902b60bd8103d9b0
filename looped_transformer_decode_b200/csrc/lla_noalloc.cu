// Decode attention for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they run decode: code that executes inside an allocator-free region of a
// host runtime, plugins that are handed only input and output buffers, or
// runtimes that forbid allocation after start-up so that memory use stays
// fixed.  lla_decode_attn_noalloc serves them: it runs the same kernels as
// lla_decode_attn, with the split-context partials and status words held in a
// fixed-size array that this library places in device memory when it is loaded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "lla_internal.cuh"

namespace {

// Largest workspace the allocation-free variant can use: 8 MiB.  Every GPU on
// which the library is loaded holds this array until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};   // context the address belongs to

// Identifier of the calling thread's current CUDA context (0 when it cannot be
// read).  A device reset or a released and re-created primary context reloads the
// library's module, and the array may then sit at another address.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with that
// device current: once per device and context (the first call there), and again
// whenever the device's context has changed since.
int scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return lla::set_error(LLA_ERR_CUDA, "lla_decode_attn_noalloc: cudaGetDevice failed: %s",
                          cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return lla::set_error(LLA_ERR_UNSUPPORTED, "lla_decode_attn_noalloc: device %d above %d", dev,
                          kMaxDevices - 1);
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return lla::set_error(LLA_ERR_CUDA,
                            "lla_decode_attn_noalloc: cudaGetSymbolAddress failed: %s",
                            cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
    // read again: the lookup above may have created the primary context
    g_scratch_ctx[dev] = ctx ? ctx : current_context_id();
  }
  *out = g_scratch_addr[dev];
  return LLA_OK;
}

}  // namespace

extern "C" int lla_decode_attn_noalloc(const lla_cfg* cfg, const void* packed,
                                       const void* rope_table, int32_t rope_max_pos, int32_t t,
                                       int32_t B, int32_t n_cap, const int32_t* ctx_len,
                                       const float* q, const float* k_self, const float* v_self,
                                       const int32_t* positions, const int32_t* q_pos,
                                       const uint16_t* c_k, const uint16_t* c_v, float* out,
                                       int32_t* status_out, void* stream) {
  int64_t num = 0, den = 0;
  int rc = lla_ratio(cfg, &num, &den);  // validates cfg, sets the error code and message
  if (rc != LLA_OK) return rc;
  if (B < 0 || n_cap < 0)
    return lla::set_error(LLA_ERR_INVALID, "lla_decode_attn_noalloc: B and n_cap must be >= 0");
  const size_t need = lla_decode_workspace_bytes(cfg, B, n_cap);
  if (need > kNoAllocScratchBytes)
    return lla::set_error(LLA_ERR_TOO_SMALL,
                          "lla_decode_attn_noalloc: this shape needs %zu bytes of scratch but the "
                          "built-in array holds %zu; call lla_decode_attn with a caller workspace",
                          need, kNoAllocScratchBytes);
  if (status_out && (reinterpret_cast<uintptr_t>(status_out) & 3u))
    return lla::set_error(LLA_ERR_INVALID, "lla_decode_attn_noalloc: status_out misaligned");
  // Every other check of lla_decode_attn, before anything is enqueued: a rejected
  // call leaves the array (and the last call's status word) as it was.
  rc = lla::decode_check_args(cfg, packed, rope_table, rope_max_pos, t, B, n_cap, ctx_len, q,
                              k_self, v_self, positions, q_pos, c_k, c_v, out);
  if (rc != LLA_OK) return rc;
  if (B == 0) return LLA_OK;   // nothing to compute; status_out is not written
  void* ws = nullptr;
  rc = scratch_address(&ws);
  if (rc != LLA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents; the two status words must
  // start at zero.  The partials are fully written before they are read.
  cudaError_t e = cudaMemsetAsync(ws, 0, 2 * sizeof(int32_t), s);
  if (e != cudaSuccess)
    return lla::set_error(LLA_ERR_CUDA, "lla_decode_attn_noalloc: clearing status: %s",
                          cudaGetErrorString(e));
  rc = lla_decode_attn(cfg, packed, rope_table, rope_max_pos, t, B, n_cap, ctx_len, q, k_self,
                       v_self, positions, q_pos, c_k, c_v, out, ws, kNoAllocScratchBytes, stream);
  if (rc != LLA_OK) return rc;
  if (status_out) {
    e = cudaMemcpyAsync(status_out, static_cast<char*>(ws) + sizeof(int32_t), sizeof(int32_t),
                        cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess)
      return lla::set_error(LLA_ERR_CUDA, "lla_decode_attn_noalloc: copying status: %s",
                            cudaGetErrorString(e));
  }
  return LLA_OK;
}
