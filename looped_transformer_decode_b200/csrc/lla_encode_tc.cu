// Encode on the 5th-generation tensor cores (sm_100a): c = x W_down - mu W_down,
// rounded to bf16 and written to each token's cache slot (gist.science,
// Kernmechanismus: latent storage; close reading §二.6 for LLA-2D).
//
// The work is a list of items (token tile of 128 or 256 tokens, latent l, K or V),
// latent fastest, so the items in flight at any moment cover a few token tiles
// completely and every token row is streamed from DRAM once.  Each item is the GEMM
//   D[tokens x r] = X[tokens x W] * W_down^T[W x r]       (W = T d, or T H d for LLA-2D)
// over W in chunks of kc = 64 (or 32) elements.  One persistent CTA per SM walks
// the items with three roles:
//   * warp 0 (one thread) streams each chunk of x with TMA (swizzled K-major boxes;
//     the per-head x is addressed as a 4-D tensor [tokens][T][H][d], so a head's
//     loop-major row needs no copy) and the matching W_down^T tile, pre-swizzled at
//     pack time, with one bulk copy, into a ring that runs on across items.  TMA
//     throughput here is set per CTA by the rows of its boxes, so W_down costs no
//     TMA rows and two CTAs share each SM when their accumulators fit;
//   * warp 1 (one thread) issues tcgen05.mma (M = 128 per 128-token sub-tile, the
//     sub-tiles sharing the W_down chunk; N = r rounded up to 16; K = 16) into one
//     of two fp32 TMEM accumulators and frees each stage with a commit;
//   * warps 2-5 drain the other accumulator meanwhile: subtract the bias (mu W_down,
//     computed with the same bf16 W_down), round to bf16 and store each token's row
//     to its slot.  Tokens past n_tok are never stored; slots outside the cache set
//     LLA_STATUS_SLOT_RANGE and are skipped.
// Waits are bounded; a timeout sets LLA_STATUS_TIMEOUT and the CTA drains and exits.
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>

#include "lla_internal.cuh"
#include "lla_sm100.cuh"

namespace lla {

namespace {

using namespace sm100;

constexpr int kEncThreads = 192;    // producer warp, MMA warp, 4 epilogue warps
constexpr int kEncMaxStages = 12;
constexpr int kEncTile = 128;       // tokens per M = 128 sub-tile
constexpr uint32_t kEncTmemCols = 512;

struct EncParams {
  int T, H, d, L, W, r_k, r_v;
  int kc;                 // K chunk (elements): 64 or 32
  int nchunks;            // W / kc
  int swz;                // descriptor swizzle code for kc
  int stages;             // ring depth
  int msub;               // 128-token sub-tiles per item: 1 or 2
  int acc_cols;           // TMEM columns of one accumulator buffer
  int nbuf;               // accumulator buffers: 2 (epilogue overlaps the next item) or 1
  uint32_t tmem_cols;     // TMEM columns allocated by one CTA
  int per_head;
  uint32_t st_bytes;      // ring stage: msub A boxes, then the B box (1 KB aligned)
  int64_t n_tok, n_slots;
  int64_t n_items;        // token tiles x 2 x L
  const int64_t* slot;
  const __nv_bfloat16* wimg_k;   // [L][nchunks][N_k][kc] operand images
  const __nv_bfloat16* wimg_v;
  const float* bias_k;    // [L][r_k]
  const float* bias_v;    // [L][r_v]
  __nv_bfloat16* ck;
  __nv_bfloat16* cv;
  int32_t* status;
};

struct Item {
  int l, kv, r, N, msub;
  int64_t tok0;
};

__device__ __forceinline__ Item decode_item(const EncParams& p, int64_t item) {
  Item it;
  it.l = (int)(item % p.L);
  it.kv = (int)((item / p.L) & 1);
  it.tok0 = (item / (2 * p.L)) * p.msub * kEncTile;
  it.r = it.kv ? p.r_v : p.r_k;
  it.N = (it.r + 15) / 16 * 16;
  // Sub-tiles wholly past n_tok are neither loaded nor multiplied.
  const int64_t left = (p.n_tok - it.tok0 + kEncTile - 1) / kEncTile;
  it.msub = left < p.msub ? (int)left : p.msub;
  return it;
}

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

// Give an async completion a bounded time (used only on the abort path).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity) && global_timer_ns() - t0 < kWaitTimeoutNs) {
  }
}

// Grid: min(items, SMs) persistent CTAs; one per SM (the CTA takes all of TMEM).
__global__ void __launch_bounds__(kEncThreads, 1)
    encode_tc_kernel(const __grid_constant__ CUtensorMap map_xk,
                     const __grid_constant__ CUtensorMap map_xv,
                     const __grid_constant__ EncParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + p.stages * p.st_bytes);
  uint64_t* empty = full + p.stages;
  uint64_t* acc_full = empty + p.stages;   // [2] MMA -> epilogue
  uint64_t* acc_empty = acc_full + 2;      // [2] epilogue (4 warps) -> MMA
  uint64_t* fin = acc_empty + 2;           // every MMA of this CTA has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t a_sub = kEncTile * p.kc * 2;
  const uint32_t a_bytes = a_sub * p.msub;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------------- producer
      tma_prefetch_desc(&map_xk);
      tma_prefetch_desc(&map_xv);
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued = 0;
      bool ok = true;
      for (int64_t item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const Item it = decode_item(p, item);
        const CUtensorMap* mx = it.kv ? &map_xv : &map_xk;
        const uint32_t b_bytes = (uint32_t)it.N * p.kc * 2;
        const __nv_bfloat16* img = (it.kv ? p.wimg_v : p.wimg_k) +
                                   (size_t)it.l * p.nchunks * it.N * p.kc;
        const uint32_t tx = a_sub * it.msub + b_bytes;
        for (int c = 0; c < p.nchunks; ++c) {
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          unsigned char* st = sm + s * p.st_bytes;
          mbar_arrive_expect_tx(&full[s], tx);
          const int k0 = c * p.kc;
          for (int j = 0; j < it.msub; ++j) {
            const int tj = (int)(it.tok0 + j * kEncTile);
            if (p.per_head)   // chunk k0 of head l: loop k0 / d, entries k0 % d + [0, kc)
              tma_load_4d(st + j * a_sub, mx, &full[s], k0 % p.d, it.l, k0 / p.d, tj);
            else
              tma_load_2d(st + j * a_sub, mx, &full[s], k0, tj);
          }
          bulk_load(st + a_bytes, img + (size_t)c * it.N * p.kc, b_bytes, &full[s]);
          ++issued;
          if (++s == p.stages) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {
        // The last `stages` loads may still be landing in shared memory.
        for (uint32_t j = 0; j < (uint32_t)p.stages && j < issued; ++j) {
          const uint32_t i = issued - 1 - j;
          drain_wait(&full[i % p.stages], (i / p.stages) & 1);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // -------------------------------------------------------------- MMA issuer
      const uint32_t sbo = 16u * p.kc;   // 8 rows of one swizzled kc-element row
      int s = 0;
      uint32_t ph = 0;
      uint32_t n = 0;
      bool ok = true;
      for (int64_t item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++n) {
        const Item it = decode_item(p, item);
        const uint32_t b = n % p.nbuf;
        if (!mbar_wait(&acc_empty[b], ((n / p.nbuf) & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * p.acc_cols;
        const uint32_t idesc = idesc_bf16_f32(128, it.N);
        for (int c = 0; c < p.nchunks; ++c) {
          if (!mbar_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(sm + s * p.st_bytes);
          const uint32_t b_addr = a_addr + a_bytes;
          for (int kk = 0; kk < p.kc / 16; ++kk) {
            const uint64_t bd = smem_desc(b_addr + kk * 32, 16, sbo, p.swz);
            for (int j = 0; j < it.msub; ++j)
              mma_bf16(d_tmem + j * it.N, smem_desc(a_addr + j * a_sub + kk * 32, 16, sbo, p.swz),
                       bd, idesc, (c > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
          if (++s == p.stages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (ok) mma_commit(&acc_full[b]);
      }
      // Also after an abort: TMEM is released only once the MMAs issued have finished.
      mma_commit(fin);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;            // TMEM lanes 32q .. 32q + 31 belong to this warp
    uint32_t n = 0;
    for (int64_t item = blockIdx.x; item < p.n_items; item += gridDim.x, ++n) {
      const Item it = decode_item(p, item);
      const uint32_t b = n % p.nbuf;
      const bool got =
          __all_sync(0xffffffffu, mbar_wait(&acc_full[b], (n / p.nbuf) & 1, abort_flag));
      if (!got) break;
      tc_fence_after();
      const float* bias = (it.kv ? p.bias_v : p.bias_k) + (size_t)it.l * it.r;
      __nv_bfloat16* cache = it.kv ? p.cv : p.ck;
      for (int j = 0; j < it.msub; ++j) {
        const int64_t tok = it.tok0 + j * kEncTile + q * 32 + lane;
        int64_t sl = -1;
        if (tok < p.n_tok) {
          sl = p.slot[tok];
          if (sl < 0 || sl >= p.n_slots) {
            if (it.l == 0 && it.kv == 0 && p.status) atomicOr(p.status, LLA_STATUS_SLOT_RANGE);
            sl = -1;
          }
        }
        __nv_bfloat16* dst = sl >= 0 ? cache + ((size_t)sl * p.L + it.l) * it.r : nullptr;
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + b * p.acc_cols + j * it.N;
        for (int c0 = 0; c0 < it.N; c0 += 16) {
          float v[16];
          tmem_ld16(taddr + c0, v);
          tmem_wait_ld();
          if (dst) {
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
              const int m0 = c0 + 8 * h8;
              if (m0 < it.r) {
                __align__(16) __nv_bfloat16 o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                  o[e] = __float2bfloat16_rn(v[8 * h8 + e] - bias[m0 + e]);
                *reinterpret_cast<uint4*>(dst + m0) = *reinterpret_cast<const uint4*>(o);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    // Normally complete already; after an abort, wait (bounded) for in-flight MMAs.
    if (lane == 0) drain_wait(fin, 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
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
  // A K chunk must not straddle two heads' rows (per head) and must tile W; the
  // packed operand images are cut with the same width.
  p.kc = encode_kc(c);
  p.swz = p.kc == 64 ? 2 : 4;
  p.nchunks = L.W / p.kc;
  const int n_k = (c.r_k + 15) / 16 * 16, n_v = (c.r_v + 15) / 16 * 16;
  const int n_max = n_k > n_v ? n_k : n_v;
  const int sms = sm_count();
  // Two CTAs per SM when each can hold two accumulators in half of TMEM.
  int cps = 2 * n_max <= (int)kEncTmemCols / 2 ? 2 : 1;
  const char* cps_env = std::getenv("LLA_ENC_CPS");
  if (cps_env && (*cps_env == '1' || (*cps_env == '2' && n_max <= (int)kEncTmemCols / 2)))
    cps = *cps_env - '0';
  p.tmem_cols = kEncTmemCols / cps;
  p.msub = 1;
  const char* ms = std::getenv("LLA_ENC_MSUB");
  if (ms && *ms == '2' && 2 * n_max <= (int)p.tmem_cols) p.msub = 2;
  p.acc_cols = p.msub * n_max;
  p.nbuf = 2 * p.acc_cols <= (int)p.tmem_cols ? 2 : 1;
  p.st_bytes = align1k(kEncTile * p.kc * 2 * p.msub + (uint32_t)n_max * p.kc * 2);
  const uint32_t tail = (2 * kEncMaxStages + 5) * 8 + 16 + 1024;   // barriers, slots, alignment
  const uint32_t max_smem = cps == 2 ? 232448u / 2 - 1024u : 232448u;
  int stages = (int)((max_smem - tail) / p.st_bytes);
  if (stages > kEncMaxStages) stages = kEncMaxStages;
  const char* st_env = std::getenv("LLA_ENC_STAGES");
  if (st_env && std::atoi(st_env) >= 2 && std::atoi(st_env) < stages) stages = std::atoi(st_env);
  if (stages < 2) return cudaErrorNotSupported;
  p.stages = stages;
  uint32_t smem = p.stages * p.st_bytes + tail;
  // Enough shared memory that no more CTAs share an SM than TMEM can hold.
  const uint32_t floor_smem = 233472u / (uint32_t)(cps + 1) + 16u;
  if (smem < floor_smem) smem = floor_smem;
  p.n_tok = n_tok;
  p.n_slots = n_slots;
  const int64_t tiles = (n_tok + (int64_t)kEncTile * p.msub - 1) / ((int64_t)kEncTile * p.msub);
  p.n_items = tiles * 2 * L.L;
  p.slot = slot;
  p.wimg_k = reinterpret_cast<const __nv_bfloat16*>(packed + L.wimgk);
  p.wimg_v = reinterpret_cast<const __nv_bfloat16*>(packed + L.wimgv);
  p.bias_k = reinterpret_cast<const float*>(packed + L.biask);
  p.bias_v = reinterpret_cast<const float*>(packed + L.biasv);
  p.ck = ck;
  p.cv = cv;
  p.status = status;

  const CUtensorMapSwizzle swz = p.kc == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap mxk, mxv;
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
  cudaError_t e = cudaFuncSetAttribute(encode_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = p.n_items < (int64_t)cps * sms ? (int)p.n_items : cps * sms;
  encode_tc_kernel<<<grid, kEncThreads, smem, s>>>(mxk, mxv, p);
  return cudaGetLastError();
}

}  // namespace lla
