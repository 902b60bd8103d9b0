// Full-memory fast path of LLA decode: the loop-t history K/V rebuilt once from
// the latents into a full bf16 cache (keys rotated at their positions), and
// ordinary decode attention over that cache.
//
// "Looped Latent Attention: 跨循环 KV 压缩精读" (cc.laoqi.cc close reading),
// §四.9, Table 5 (the "full-memory fast path" latency row) and the paragraph
// after it: the fast path keeps the complete rebuilt K/V instead of rebuilding
// on every read, so it gives up the cache saving; §二.3: the codec works on
// pre-RoPE K, and the model rotates the rebuilt key at its position before
// caching it.
//
// Layout of the full cache (one loop): K and V each bf16 [B][H][n_cap][d],
// head-major, so one (sequence, head) history is a contiguous run of rows.
//
// full_rebuild_kernel   (CUDA cores) x^ = c W_up,t^T + mu_t, K rotated, bf16 store.
//                        Runs once per token (or once over a history); not on the
//                        per-step path.
// full_decode_kernel<D>  the per-step path: persistent CTAs stream 64-token K/V
//                        tiles through a TMA ring (one producer warp, 8 consumer
//                        warps); each consumer warp keeps its own online softmax
//                        over 8 rows of every tile, and the warps merge at the end
//                        of each (sequence, head, split) item.  HBM-bound: 2 d
//                        bf16 per token and head against 2 d FMAs.
// full_combine_kernel<D> merges the splits and the in-flight token when a head has
//                        more than one split.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <vector>

#include "lla_internal.cuh"
#include "lla_sm100.cuh"

namespace lla {
namespace {

using namespace sm100;

// ---------------------------------------------------------------- rebuild once

constexpr int kRecRows = 8;   // rows of one register block

// grid (row groups, H, 2): z = 0 rebuilds and rotates K, z = 1 rebuilds V.
// blockDim.x = d: thread i owns output dimension i.  The up-projection of head h
// at loop t is staged in shared memory as [r][d] so a warp reads consecutive
// words (W_up,k is packed [d][r_k] and transposed here; W_up,v is packed [r_v][d]).
__global__ void __launch_bounds__(128) full_rebuild_kernel(FullRebuildArgs a) {
  extern __shared__ float smf[];
  const int d = a.d, h = blockIdx.y, i = threadIdx.x;
  const bool is_k = blockIdx.z == 0;
  const int r = is_k ? a.r_k : a.r_v;
  float* w = smf;                          // [r][d]
  float* lat = w + r * d;                  // [kRecRows][r]
  float* x = lat + kRecRows * r;           // [kRecRows][d] rebuilt K before rotation
  // 16-byte loads, four in flight per thread (d r is a multiple of 32)
  if (is_k) {
    const float4* wg = reinterpret_cast<const float4*>(a.wupk_t + (size_t)h * d * r);   // [d][r]
    const int n4 = d * r / 4;
    for (int b4 = i; b4 < n4; b4 += 4 * d) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (b4 + u * d < n4) v[u] = __ldg(wg + b4 + u * d);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (b4 + u * d >= n4) break;
        const int idx = 4 * (b4 + u * d), row = idx / r, k = idx % r;   // r % 4 == 0
        w[k * d + row] = v[u].x;
        w[(k + 1) * d + row] = v[u].y;
        w[(k + 2) * d + row] = v[u].z;
        w[(k + 3) * d + row] = v[u].w;
      }
    }
  } else {
    const float4* wg = reinterpret_cast<const float4*>(a.wupv_t + (size_t)h * r * d);   // [r][d]
    float4* w4 = reinterpret_cast<float4*>(w);
    const int n4 = d * r / 4;
    for (int b4 = i; b4 < n4; b4 += 4 * d) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (b4 + u * d < n4) v[u] = __ldg(wg + b4 + u * d);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (b4 + u * d < n4) w4[b4 + u * d] = v[u];
    }
  }
  const float mu = (is_k ? a.muk_t : a.muv_t)[(size_t)h * d + i];
  const __nv_bfloat16* lat_g = is_k ? a.ck : a.cv;
  const long long lat_tok = is_k ? a.lat_tok_k : a.lat_tok_v;
  const long long lat_head = is_k ? a.lat_head_k : a.lat_head_v;
  __nv_bfloat16* dst = is_k ? a.k_full : a.v_full;
  const long long n_slots = (long long)a.B * a.n_cap;
  const int half = d / 2;
  __syncthreads();

  for (long long row0 = (long long)blockIdx.x * kRecRows; row0 < a.n_rows;
       row0 += (long long)gridDim.x * kRecRows) {
    long long slot[kRecRows];
#pragma unroll
    for (int rr = 0; rr < kRecRows; ++rr) {
      const long long row = row0 + rr;
      long long s = -1;
      if (row < a.n_rows) {
        s = a.slot ? a.slot[row] : row;
        if (s < 0 || s >= n_slots) {
          if (i == 0 && is_k && h == 0 && a.status) atomicOr(a.status, LLA_STATUS_SLOT_RANGE);
          s = -1;
        }
      }
      slot[rr] = s;
      for (int k = i; k < r; k += d)
        lat[rr * r + k] = s >= 0 ? __bfloat162float(lat_g[s * lat_tok + h * lat_head + k]) : 0.f;
    }
    __syncthreads();
    float acc[kRecRows];
#pragma unroll
    for (int rr = 0; rr < kRecRows; ++rr) acc[rr] = mu;
    for (int k = 0; k < r; ++k) {
      const float wk = w[k * d + i];
#pragma unroll
      for (int rr = 0; rr < kRecRows; ++rr) acc[rr] = fmaf(lat[rr * r + k], wk, acc[rr]);
    }
    if (is_k) {
#pragma unroll
      for (int rr = 0; rr < kRecRows; ++rr) x[rr * d + i] = acc[rr];
      __syncthreads();
      const int pi = i < half ? i : i - half;
#pragma unroll
      for (int rr = 0; rr < kRecRows; ++rr) {
        if (slot[rr] < 0) continue;
        int pos = a.positions[slot[rr]];
        if (pos < 0 || pos >= a.rope_max_pos) {
          if (i == 0 && h == 0 && a.status) atomicOr(a.status, LLA_STATUS_POSITION_RANGE);
          pos = pos < 0 ? 0 : a.rope_max_pos - 1;
        }
        const float2 cs = a.rope[(size_t)pos * half + pi];
        const float lo = x[rr * d + pi], hi = x[rr * d + pi + half];
        acc[rr] = i < half ? lo * cs.x - hi * cs.y : lo * cs.y + hi * cs.x;
      }
    }
#pragma unroll
    for (int rr = 0; rr < kRecRows; ++rr) {
      if (slot[rr] < 0) continue;
      const long long b = slot[rr] / a.n_cap, j = slot[rr] % a.n_cap;
      dst[((b * a.H + h) * a.n_cap + j) * d + i] = __float2bfloat16_rn(acc[rr]);
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- decode

constexpr int kFullTile = 64;                   // history tokens per tile
constexpr int kFullWarps = 8;                   // consumer warps (8 tokens of a tile each)
constexpr int kFullThreads = 32 * (1 + kFullWarps);

template <int D>
struct FullShape {
  static constexpr int kBoxD = D % 64 == 0 ? 64 : 32;   // dims per TMA box: 128- or 64-byte rows
  static constexpr int kBoxes = D / kBoxD;               // boxes per K (or V) tile
  static constexpr int kChunks = D / 32;                 // 16-byte chunks per lane per row
  static constexpr uint32_t kBoxBytes = kFullTile * kBoxD * 2;
  static constexpr uint32_t kTileBytes = kBoxes * kBoxBytes;
  static constexpr uint32_t kStageBytes = 2 * kTileBytes;   // K tile, then V tile
  // 64-byte box rows stream at full rate only with two CTAs per SM
  static constexpr int kCtasPerSm = kBoxD == 64 ? 1 : 2;
  static constexpr int kStages =
      kCtasPerSm == 1 ? (196608 / kStageBytes > 8 ? 8 : 196608 / kStageBytes)
                      : (98304 / kStageBytes > 8 ? 8 : 98304 / kStageBytes);
  // shared memory: stages (1024-aligned), merge buffer, barriers, misc
  static constexpr uint32_t kMergeOff = kStages * kStageBytes;
  static constexpr uint32_t kBarOff = kMergeOff + kFullWarps * (D + 2) * 4;
  static constexpr uint32_t kMiscOff = kBarOff + 2 * kStages * 8;
  static constexpr uint32_t kSmemBytes = kMiscOff + 16 + 1024;
};

// Byte offset of 16-byte chunk c (8 dims) of tile row `row` in a K or V tile staged
// by the TMA with the swizzle of its box width (128-byte rows: chunk ^ (row & 7);
// 64-byte rows: chunk ^ ((row >> 1) & 3)).
template <int D>
__device__ __forceinline__ uint32_t full_chunk_off(int row, int c) {
  using S = FullShape<D>;
  if constexpr (S::kBoxD == 64) {
    return (c >> 3) * S::kBoxBytes + row * 128 + (((c & 7) ^ (row & 7)) << 4);
  } else {
    return (c >> 2) * S::kBoxBytes + row * 64 + (((c & 3) ^ ((row >> 1) & 3)) << 4);
  }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
      : "memory");
}

// bar.sync over `threads` threads that also ORs `pred` across them.
__device__ __forceinline__ bool named_barrier_or(uint32_t id, uint32_t threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void bf16x8_to_float(const uint4 u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = __uint_as_float(w[k] << 16);
    f[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
}

struct FullItem {
  int b, h, s, tok0, tok_end, ntiles;
};

__device__ __forceinline__ FullItem full_item(const FullDecodeParams& p, int item, bool flag) {
  FullItem r;
  r.s = item % p.S;
  const int u = item / p.S;
  r.h = u % p.H;
  r.b = u / p.H;
  int n = p.ctx_len[r.b];
  if (n < 0 || n > p.n_cap) {
    if (flag) atomicOr(p.status, LLA_STATUS_CTX_RANGE);
    n = n < 0 ? 0 : p.n_cap;
  }
  r.tok0 = r.s * p.tps * kFullTile;
  r.tok_end = min(r.tok0 + p.tps * kFullTile, n);
  r.ntiles = r.tok_end > r.tok0 ? (r.tok_end - r.tok0 + kFullTile - 1) / kFullTile : 0;
  return r;
}

// Warp roles: warp 0 lane 0 issues the TMA loads; warps 1..8 consume.  Consumer
// lane (g = lane & 7, p = lane >> 3) owns tile row 8 w + g and the 16-byte chunks
// p, p + 4, ... of that row, so a quarter-warp of one load instruction touches
// eight rows at one logical chunk, which the swizzle spreads over all 32 banks.
template <int D>
__global__ void __launch_bounds__(kFullThreads, FullShape<D>::kCtasPerSm)
    full_decode_kernel(const __grid_constant__ CUtensorMap mk,
                       const __grid_constant__ CUtensorMap mv, const FullDecodeParams p) {
  using S = FullShape<D>;
  constexpr int NK = S::kChunks;
  constexpr int NST = S::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* merge = reinterpret_cast<float*>(sm + S::kMergeOff);   // [8][2 + D]
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + S::kBarOff);
  uint64_t* empty = full + NST;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + S::kMiscOff);
  float* self_s = reinterpret_cast<float*>(sm + S::kMiscOff + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kFullWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&mk);
      tma_prefetch_desc(&mv);
      uint32_t it = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const FullItem r = full_item(p, item, false);
        const int row0 = (r.b * p.H + r.h) * p.n_cap + r.tok0;
        for (int k = 0; k < r.ntiles; ++k, ++it) {
          const uint32_t stage = it % NST, ph = (it / NST) & 1u;
          if (!mbar_wait(&empty[stage], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], S::kStageBytes);
          unsigned char* st = sm + stage * S::kStageBytes;
#pragma unroll
          for (int bx = 0; bx < S::kBoxes; ++bx)
            tma_load_2d(st + bx * S::kBoxBytes, &mk, &full[stage], bx * S::kBoxD,
                        row0 + k * kFullTile);
#pragma unroll
          for (int bx = 0; bx < S::kBoxes; ++bx)
            tma_load_2d(st + S::kTileBytes + bx * S::kBoxBytes, &mv, &full[stage], bx * S::kBoxD,
                        row0 + k * kFullTile);
        }
      }
      if (!ok) {
        // consumers stopped: let the copies already issued land before the CTA exits
        for (uint32_t j = 0; j < (uint32_t)NST && j < it; ++j) {
          const uint32_t i2 = it - 1 - j;
          const unsigned long long t0 = global_timer_ns();
          while (!mbar_try_wait(&full[i2 % NST], (i2 / NST) & 1u) &&
                 global_timer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ consumers
    const int cw = warp - 1, g = lane & 7, pp = lane >> 3;
    const int row = cw * 8 + g;                // tile row of this lane
    const int et = threadIdx.x - 32;           // 0 .. 255
    const int half = D / 2;
    uint32_t it = 0;
    bool aborted = false;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
      const FullItem r = full_item(p, item, et == 0);
      const size_t bh = (size_t)r.b * p.H + r.h;
      int qp = p.q_pos[r.b];
      if (qp < 0 || qp >= p.rope_max_pos) {
        if (et == 0) atomicOr(p.status, LLA_STATUS_POSITION_RANGE);
        qp = qp < 0 ? 0 : p.rope_max_pos - 1;
      }
      // kappa * RoPE(q, q_pos) on this lane's dims
      const float* qg = p.q + bh * D;
      const float2* rope_q = p.rope + (size_t)qp * half;
      float qr[NK][8];
#pragma unroll
      for (int kk = 0; kk < NK; ++kk) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int dim = (pp + 4 * kk) * 8 + e;
          const int pi = dim < half ? dim : dim - half;
          const float2 cs = __ldg(rope_q + pi);
          const float lo = __ldg(qg + pi), hi = __ldg(qg + pi + half);
          qr[kk][e] = p.kappa * (dim < half ? lo * cs.x - hi * cs.y : lo * cs.y + hi * cs.x);
        }
      }
      if (p.fuse && cw == 0) {
        // the in-flight token sits at q_pos too, so its score needs no rotation
        float acc = 0.f;
        for (int dd = lane; dd < D; dd += 32) acc = fmaf(qg[dd], p.k_self[bh * D + dd], acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) *self_s = p.kappa * acc;
      }
      float m = -INFINITY, l = 0.f;
      float o[NK][8];
#pragma unroll
      for (int kk = 0; kk < NK; ++kk)
#pragma unroll
        for (int e = 0; e < 8; ++e) o[kk][e] = 0.f;

      for (int k = 0; !aborted && k < r.ntiles; ++k, ++it) {
        const uint32_t stage = it % NST, ph = (it / NST) & 1u;
        if (!mbar_wait(&full[stage], ph, abort_flag)) {
          aborted = true;
          break;
        }
        const unsigned char* kt = sm + stage * S::kStageBytes;
        const unsigned char* vt = kt + S::kTileBytes;
        const int cnt = min(kFullTile, r.tok_end - (r.tok0 + k * kFullTile));
        const bool valid = row < cnt;
        float s = 0.f;
        if (valid) {
#pragma unroll
          for (int kk = 0; kk < NK; ++kk) {
            float kf[8];
            bf16x8_to_float(*reinterpret_cast<const uint4*>(kt + full_chunk_off<D>(row, pp + 4 * kk)),
                            kf);
#pragma unroll
            for (int e = 0; e < 8; ++e) s = fmaf(qr[kk][e], kf[e], s);
          }
        }
        s += __shfl_xor_sync(0xffffffffu, s, 8);
        s += __shfl_xor_sync(0xffffffffu, s, 16);
        if (!valid) s = -INFINITY;
        float mt = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, 1));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
        if (mt > m) {                          // warp-uniform
          const float sc = exp2f(m - mt);      // 0 on the first tile (m = -inf)
          l *= sc;
#pragma unroll
          for (int kk = 0; kk < NK; ++kk)
#pragma unroll
            for (int e = 0; e < 8; ++e) o[kk][e] *= sc;
          m = mt;
        }
        if (valid) {
          const float w = exp2f(s - m);
          l += w;
#pragma unroll
          for (int kk = 0; kk < NK; ++kk) {
            float vf[8];
            bf16x8_to_float(*reinterpret_cast<const uint4*>(vt + full_chunk_off<D>(row, pp + 4 * kk)),
                            vf);
#pragma unroll
            for (int e = 0; e < 8; ++e) o[kk][e] = fmaf(w, vf[e], o[kk][e]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
      }
      // warp partial: sum over the 8 rows (lanes with equal pp)
#pragma unroll
      for (int sh = 1; sh < 8; sh <<= 1) {
        l += __shfl_xor_sync(0xffffffffu, l, sh);
#pragma unroll
        for (int kk = 0; kk < NK; ++kk)
#pragma unroll
          for (int e = 0; e < 8; ++e) o[kk][e] += __shfl_xor_sync(0xffffffffu, o[kk][e], sh);
      }
      float* mw = merge + cw * (D + 2);
      if (g == 0) {
#pragma unroll
        for (int kk = 0; kk < NK; ++kk)
#pragma unroll
          for (int e = 0; e < 8; ++e) mw[2 + (pp + 4 * kk) * 8 + e] = o[kk][e];
        if (pp == 0) {
          mw[0] = m;
          mw[1] = l;
        }
      }
      named_barrier(1, 32 * kFullWarps);
      if (et < D) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kFullWarps; ++w) M = fmaxf(M, merge[w * (D + 2)]);
        float L = 0.f, O = 0.f;
        if (M > -INFINITY) {
#pragma unroll
          for (int w = 0; w < kFullWarps; ++w) {
            const float mwv = merge[w * (D + 2)];
            const float f = mwv > -INFINITY ? exp2f(mwv - M) : 0.f;
            L = fmaf(merge[w * (D + 2) + 1], f, L);
            O = fmaf(merge[w * (D + 2) + 2 + et], f, O);
          }
        }
        if (p.fuse) {
          const float ss = *self_s;
          const float ms = fmaxf(M, ss);
          const float fa = M > -INFINITY ? exp2f(M - ms) : 0.f, fs = exp2f(ss - ms);
          p.out[bh * D + et] = (O * fa + fs * p.v_self[bh * D + et]) / (L * fa + fs);
        } else {
          float* part = p.partials + (bh * p.S + r.s) * (D + 2);
          if (et == 0) {
            part[0] = M;
            part[1] = L;
          }
          part[2 + et] = O;
        }
      }
      // every consumer warp leaves together when any of them gave up
      if (named_barrier_or(1, 32 * kFullWarps, aborted || *abort_flag)) {
        aborted = true;
        break;
      }
    }
    if (aborted && et == 0) atomicOr(p.status, LLA_STATUS_TIMEOUT);
  }
  // the last CTA to finish publishes the call's status word and re-arms the counter
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.counter, 1u) == gridDim.x - 1) {
      __threadfence();
      p.status[1] = atomicExch(&p.status[0], 0);
      atomicExch(p.counter, 0u);
    }
  }
}

// One block of D threads per (b, h): merge the S split partials with the in-flight
// token (score kappa q . k_self, both at q_pos) and normalise.
template <int D>
__global__ void __launch_bounds__(128) full_combine_kernel(const FullDecodeParams p) {
  __shared__ float red[4];
  const size_t bh = blockIdx.x;
  const int i = threadIdx.x;
  float acc = p.q[bh * D + i] * p.k_self[bh * D + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((i & 31) == 0) red[i >> 5] = acc;
  __syncthreads();
  float ss = 0.f;
  for (int w = 0; w < D / 32; ++w) ss += red[w];
  ss *= p.kappa;
  const float* part = p.partials + bh * p.S * (D + 2);
  float M = ss;
  for (int s = 0; s < p.S; ++s) M = fmaxf(M, part[s * (D + 2)]);
  const float fs = exp2f(ss - M);
  float L = fs, O = fs * p.v_self[bh * D + i];
  for (int s = 0; s < p.S; ++s) {
    const float ms = part[s * (D + 2)];
    if (!(ms > -INFINITY)) continue;
    const float f = exp2f(ms - M);
    L = fmaf(part[s * (D + 2) + 1], f, L);
    O = fmaf(part[s * (D + 2) + 2 + i], f, O);
  }
  p.out[bh * D + i] = O / L;
}

bool make_full_map(CUtensorMap* map, const void* base, int D, long long rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const int boxd = D % 64 == 0 ? 64 : 32;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {(cuuint32_t)boxd, (cuuint32_t)kFullTile};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  boxd == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_full_decode_t(const FullDecodeParams& p, const void* k_full,
                                 const void* v_full, int grid, cudaStream_t s) {
  using S = FullShape<D>;
  CUtensorMap mk, mv;
  // with no history no tile is loaded, and one row keeps the maps well formed
  const long long rows = std::max(1LL, (long long)p.B * p.H * p.n_cap);
  if (!make_full_map(&mk, k_full, D, rows) || !make_full_map(&mv, v_full, D, rows))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(full_decode_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmemBytes);
  if (e != cudaSuccess) return e;
  full_decode_kernel<D><<<grid, kFullThreads, S::kSmemBytes, s>>>(mk, mv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.fuse) return e;
  full_combine_kernel<D><<<p.B * p.H, D, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

// Split plan: S context splits per (b, h) minimising the busiest CTA's cost when
// the B H S items are dealt round-robin to the persistent grid; an item costs its
// 64-token tiles plus one tile of start/finish work, and S > 1 adds the combine.
FullPlan full_plan(const lla_cfg& c, int B, int n_cap) {
  FullPlan pl;
  const int D = c.d_head;
  const int per_sm = D % 64 == 0 ? 1 : 2;
  pl.grid_max = sm_count() * per_sm;
  const int n_tiles = std::max(1, (n_cap + kFullTile - 1) / kFullTile);
  const long long units = (long long)B * c.H;
  if (units <= 0) return pl;
  constexpr double kItemCost = 1.0, kCombineCost = 1.0;   // in tiles
  const int grid = pl.grid_max;
  int s_max = (int)std::max<long long>(1, (4 * grid + units - 1) / units);
  s_max = std::min(std::min(s_max, kMaxSplits), n_tiles);
  double best = 1e300;
  int best_s = 1;
  for (int S = 1; S <= s_max; ++S) {
    const int tpi = (n_tiles + S - 1) / S;
    const int s_eff = (n_tiles + tpi - 1) / tpi;
    const long long items = units * s_eff;
    double worst = 0.0;
    if (items > grid) {
      std::vector<double> cta(grid, 0.0);
      for (long long it = 0; it < items; ++it)
        cta[it % grid] += std::min(tpi, n_tiles - (int)(it % s_eff) * tpi) + kItemCost;
      for (double v : cta) worst = std::max(worst, v);
    } else {
      worst = tpi + kItemCost;
    }
    const double cost = worst + (s_eff > 1 ? kCombineCost : 0.0);
    if (cost < best - 1e-9) {
      best = cost;
      best_s = s_eff;
    }
  }
  pl.tps = (n_tiles + best_s - 1) / best_s;
  pl.S = (n_tiles + pl.tps - 1) / pl.tps;
  pl.n_items = (long long)units * pl.S;
  pl.grid = (int)std::min<long long>(pl.n_items, grid);
  return pl;
}

cudaError_t launch_full_rebuild(const FullRebuildArgs& a, cudaStream_t s) {
  if (a.n_rows <= 0) return cudaSuccess;
  const int r_max = std::max(a.r_k, a.r_v);
  const size_t smem = ((size_t)r_max * a.d + (size_t)kRecRows * (r_max + a.d)) * 4;
  cudaError_t e = cudaFuncSetAttribute(full_rebuild_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long groups = (a.n_rows + kRecRows - 1) / kRecRows;
  const int gx = (int)std::min<long long>(groups, std::max(1, 1184 / a.H));
  full_rebuild_kernel<<<dim3(gx, a.H, 2), a.d, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_full_decode(const FullDecodeParams& p, const void* k_full, const void* v_full,
                               int grid, cudaStream_t s) {
  switch (p.d) {
    case 32: return launch_full_decode_t<32>(p, k_full, v_full, grid, s);
    case 64: return launch_full_decode_t<64>(p, k_full, v_full, grid, s);
    case 96: return launch_full_decode_t<96>(p, k_full, v_full, grid, s);
    case 128: return launch_full_decode_t<128>(p, k_full, v_full, grid, s);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace lla
