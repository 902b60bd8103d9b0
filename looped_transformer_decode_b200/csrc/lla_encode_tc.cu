// Encode on the 5th-generation tensor cores (sm_100a): c = x W_down - mu W_down,
// rounded to bf16 and written to each token's cache slot (gist.science,
// Kernmechanismus: latent storage; close reading §二.6 for LLA-2D).
//
// One CTA per (tile of 128 tokens, latent l, K or V).  The GEMM is
//   D[128 tokens x r] = X[128 x W] * W_down^T[W x r]      (W = T d, or T H d for LLA-2D)
// streamed over W in chunks of KC = 64 (or 32) elements:
//   * warp 0 (one thread) loads each chunk of x and of the packed W_down^T with TMA
//     into a 4-stage ring (swizzled K-major boxes; the per-head x is addressed as
//     a 4-D tensor [tokens][T][H][d] so a head's loop-major row needs no copy);
//   * warp 1 (one thread) issues tcgen05.mma (M = 128, N = r rounded up to 16,
//     K = 16) accumulating in fp32 in TMEM and frees each stage with a commit;
//   * all four warps then read their 32 token rows from TMEM, subtract the bias
//     (mu W_down, computed with the same bf16 W_down), round to bf16 and store the
//     row to its slot.  Tokens past n_tok are never stored; slots outside the cache
//     set LLA_STATUS_SLOT_RANGE and are skipped.
// Waits are bounded; a timeout sets LLA_STATUS_TIMEOUT and the CTA drains and exits.
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>

#include "lla_internal.cuh"
#include "lla_sm100.cuh"

namespace lla {

namespace {

using namespace sm100;

constexpr int kEncThreads = 128;
constexpr int kEncMaxStages = 4;
constexpr int kEncTile = 128;

struct EncParams {
  int T, H, d, L, W, r_k, r_v;
  int kc;                 // K chunk (elements): 64 or 32
  int stages;             // ring depth, 2..kEncMaxStages
  int nchunks;            // W / kc
  int swz;                // descriptor swizzle code for kc
  int per_head;
  int64_t n_tok, n_slots;
  const int64_t* slot;
  const float* bias_k;    // [L][r_k]
  const float* bias_v;    // [L][r_v]
  __nv_bfloat16* ck;
  __nv_bfloat16* cv;
  int32_t* status;
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

// Grid: (token tiles, L, 2).  Dynamic smem: p.stages x (A chunk + B chunk) + barriers.
__global__ void __launch_bounds__(kEncThreads, 1)
    encode_tc_kernel(const __grid_constant__ CUtensorMap map_xk,
                     const __grid_constant__ CUtensorMap map_xv,
                     const __grid_constant__ CUtensorMap map_wk,
                     const __grid_constant__ CUtensorMap map_wv,
                     const __grid_constant__ EncParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tile = blockIdx.x, l = blockIdx.y, kv = blockIdx.z;
  const int r = kv ? p.r_v : p.r_k;
  const int N = (r + 15) / 16 * 16;
  const uint32_t a_bytes = kEncTile * p.kc * 2;
  const uint32_t b_bytes = (uint32_t)N * p.kc * 2;
  const uint32_t st_bytes = (a_bytes + b_bytes + 1023) / 1024 * 1024;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + p.stages * st_bytes);
  uint64_t* empty = full + p.stages;
  uint64_t* done = empty + p.stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t tcols = 32;
  while (tcols < (uint32_t)N) tcols <<= 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const CUtensorMap* mx = kv ? &map_xv : &map_xk;
  const CUtensorMap* mw = kv ? &map_wv : &map_wk;
  const int tok0 = tile * kEncTile;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- producer
    tma_prefetch_desc(mx);
    tma_prefetch_desc(mw);
    int c = 0;
    for (; c < p.nchunks; ++c) {
      const int s = c % p.stages;
      if (!mbar_wait(&empty[s], ((c / p.stages) & 1) ^ 1, abort_flag)) break;
      unsigned char* st = sm + s * st_bytes;
      mbar_arrive_expect_tx(&full[s], a_bytes + b_bytes);
      const int k0 = c * p.kc;
      if (p.per_head) {
        // x as [tokens][T][H][d]: chunk k0 of head l is loop t = k0 / d, entries i0..i0+kc
        tma_load_4d(st, mx, &full[s], k0 % p.d, l, k0 / p.d, tok0);
      } else {
        tma_load_2d(st, mx, &full[s], k0, tok0);
      }
      tma_load_2d(st + a_bytes, mw, &full[s], k0, l * r);
    }
    if (*abort_flag) {
      for (int j = 0; j < p.stages && j < c; ++j) {
        const int i = c - 1 - j;
        const unsigned long long t0 = global_timer_ns();
        while (!mbar_try_wait(&full[i % p.stages], (i / p.stages) & 1) &&
               global_timer_ns() - t0 < kWaitTimeoutNs) {
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(128, N);
    const uint32_t sbo = 16u * p.kc;   // 8 rows of one kc-element swizzled row
    for (int c = 0; c < p.nchunks; ++c) {
      const int s = c % p.stages;
      if (!mbar_wait(&full[s], (c / p.stages) & 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t a_addr = smem_addr(sm + s * st_bytes);
      const uint32_t b_addr = a_addr + a_bytes;
#pragma unroll 4
      for (int kk = 0; kk < p.kc / 16; ++kk) {
        mma_bf16(tmem_base, smem_desc(a_addr + kk * 32, 16, sbo, p.swz),
                 smem_desc(b_addr + kk * 32, 16, sbo, p.swz), idesc, (c > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(&empty[s]);
    }
    // Also after an abort: `done` then tracks the MMAs already issued, so TMEM is
    // released only once they have finished.
    mma_commit(done);
  }
  __syncwarp();

  // ------------------------------------------------------------------ epilogue
  bool ok = mbar_wait(done, 0, abort_flag);
  if (!ok) {
    // Aborted: still give the MMAs already issued a bounded time to finish.
    const unsigned long long t0 = global_timer_ns();
    while (!mbar_try_wait(done, 0) && global_timer_ns() - t0 < kWaitTimeoutNs) {
    }
  }
  ok = __all_sync(0xffffffffu, ok && !*abort_flag);
  tc_fence_after();
  const int row = warp * 32 + lane;
  const int64_t tok = (int64_t)tok0 + row;
  const float* bias = (kv ? p.bias_v : p.bias_k) + (size_t)l * r;
  __nv_bfloat16* cache = kv ? p.cv : p.ck;
  int64_t s = -1;
  if (tok < p.n_tok) {
    s = p.slot[tok];
    if (s < 0 || s >= p.n_slots) {
      if (l == 0 && kv == 0 && p.status) atomicOr(p.status, LLA_STATUS_SLOT_RANGE);
      s = -1;
    }
  }
  if (ok) {
    __nv_bfloat16* dst = s >= 0 ? cache + ((size_t)s * p.L + l) * r : nullptr;
    for (int c0 = 0; c0 < N; c0 += 16) {
      float v[16];
      tmem_ld16(tmem_base + ((uint32_t)(warp * 32) << 16) + c0, v);
      tmem_wait_ld();
      if (dst) {
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
          const int m0 = c0 + 8 * h8;
          if (m0 < r) {
            __align__(16) __nv_bfloat16 o[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = __float2bfloat16_rn(v[8 * h8 + e] - bias[m0 + e]);
            *reinterpret_cast<uint4*>(dst + m0) = *reinterpret_cast<const uint4*>(o);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tcols);
  }
  if (threadIdx.x == 0 && *abort_flag && p.status) atomicOr(p.status, LLA_STATUS_TIMEOUT);
}

uint32_t align1k(uint32_t x) { return (x + 1023u) / 1024u * 1024u; }

bool encode_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swz) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Tensor-core encode; returns cudaErrorNotSupported when the shape (or the
// LLA_ENCODE_PATH=cuda_core override) leaves it to the CUDA-core kernel.
cudaError_t launch_encode_tc(const lla_cfg& c, const PackedLayout& L, const char* packed,
                             int64_t n_tok, const __nv_bfloat16* xk, const __nv_bfloat16* xv,
                             const int64_t* slot, int64_t n_slots, __nv_bfloat16* ck,
                             __nv_bfloat16* cv, int32_t* status, cudaStream_t s) {
  const char* env = std::getenv("LLA_ENCODE_PATH");
  if (env && std::strcmp(env, "cuda_core") == 0) return cudaErrorNotSupported;
  const bool per_head = c.mode == LLA_MODE_PER_HEAD;
  EncParams p{};
  p.T = c.T;
  p.H = c.H;
  p.d = c.d_head;
  p.L = L.L;
  p.W = L.W;
  p.r_k = c.r_k;
  p.r_v = c.r_v;
  p.per_head = per_head ? 1 : 0;
  // A K chunk must not straddle two heads' rows (per head) and must tile W.
  const int unit = per_head ? c.d_head : L.W;
  p.kc = unit % 64 == 0 ? 64 : (unit % 32 == 0 ? 32 : 0);
  if (p.kc == 0) return cudaErrorNotSupported;
  p.swz = p.kc == 64 ? 2 : 4;
  p.nchunks = L.W / p.kc;
  const int n_k = (c.r_k + 15) / 16 * 16, n_v = (c.r_v + 15) / 16 * 16;
  const int n_max = n_k > n_v ? n_k : n_v;
  const uint32_t a_bytes = kEncTile * p.kc * 2;
  const uint32_t st_max = align1k(a_bytes + (uint32_t)n_max * p.kc * 2);
  // Two CTAs per SM when the ring allows it: one drains its accumulator while
  // the other streams.
  int stages = (int)(115712u / st_max);
  p.stages = stages < 2 ? 2 : (stages > kEncMaxStages ? kEncMaxStages : stages);
  uint32_t smem = p.stages * st_max + (2 * kEncMaxStages + 2) * 8 + 1024;
  // Never more CTAs on one SM than TMEM can hold at once (512 columns).
  uint32_t tcols = 32;
  while (tcols < (uint32_t)n_max) tcols <<= 1;
  const uint32_t per_sm = 512u / tcols;
  const uint32_t floor_smem = 233472u / (per_sm + 1) + 16u;
  if (smem < floor_smem) smem = floor_smem;
  if (smem > 232448u) return cudaErrorNotSupported;
  p.n_tok = n_tok;
  p.n_slots = n_slots;
  p.slot = slot;
  p.bias_k = reinterpret_cast<const float*>(packed + L.biask);
  p.bias_v = reinterpret_cast<const float*>(packed + L.biasv);
  p.ck = ck;
  p.cv = cv;
  p.status = status;

  const CUtensorMapSwizzle swz = p.kc == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap mxk, mxv, mwk, mwv;
  const uint64_t e2 = 2;
  if (per_head) {
    const cuuint64_t dims[4] = {(cuuint64_t)c.d_head, (cuuint64_t)c.H, (cuuint64_t)c.T,
                                (cuuint64_t)n_tok};
    const cuuint64_t str[3] = {e2 * c.d_head, e2 * c.d_head * c.H, e2 * c.d_head * c.H * c.T};
    const cuuint32_t box[4] = {(cuuint32_t)p.kc, 1, 1, (cuuint32_t)kEncTile};
    if (!encode_map(&mxk, xk, 4, dims, str, box, swz) ||
        !encode_map(&mxv, xv, 4, dims, str, box, swz))
      return cudaErrorNotSupported;
  } else {
    const cuuint64_t dims[2] = {(cuuint64_t)L.W, (cuuint64_t)n_tok};
    const cuuint64_t str[1] = {e2 * L.W};
    const cuuint32_t box[2] = {(cuuint32_t)p.kc, (cuuint32_t)kEncTile};
    if (!encode_map(&mxk, xk, 2, dims, str, box, swz) ||
        !encode_map(&mxv, xv, 2, dims, str, box, swz))
      return cudaErrorNotSupported;
  }
  {
    const cuuint64_t str[1] = {e2 * L.W};
    const cuuint64_t dk[2] = {(cuuint64_t)L.W, (cuuint64_t)L.L * c.r_k};
    const cuuint64_t dv[2] = {(cuuint64_t)L.W, (cuuint64_t)L.L * c.r_v};
    const cuuint32_t bk[2] = {(cuuint32_t)p.kc, (cuuint32_t)n_k};
    const cuuint32_t bv[2] = {(cuuint32_t)p.kc, (cuuint32_t)n_v};
    if (!encode_map(&mwk, packed + L.wdk, 2, dk, str, bk, swz) ||
        !encode_map(&mwv, packed + L.wdv, 2, dv, str, bv, swz))
      return cudaErrorNotSupported;
  }
  cudaError_t e = cudaFuncSetAttribute(encode_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((n_tok + kEncTile - 1) / kEncTile), (unsigned)L.L, 2);
  encode_tc_kernel<<<grid, kEncThreads, smem, s>>>(mxk, mxv, mwk, mwv, p);
  return cudaGetLastError();
}

}  // namespace lla
