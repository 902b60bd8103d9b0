// CUDA-core kernels: RoPE table, codec packing, encode, and the split-context
// decode attention with its combine pass.
//
// Decode formulation (per head h, loop t; pairs i < d/2 of the split-half RoPE):
//   write a key as complex pairs  k~_i = k_i + i k_{i+d/2}; RoPE at position p
//   multiplies k~_i by e^{i p theta_i}, and the score is Re sum_i conj(q'~_i) k'~_i.
//   With k~ = c W~^T + mu~ (W~_{i,m} = W[i][m] + i W[i+d/2][m]) the query can be
//   folded into the up-projection once per (b, h):
//     A~_{m,i} = kappa conj(q'~_i) W~_{i,m},   M~_i = kappa conj(q'~_i) mu~_i
//     s_j      = Re sum_i (sum_m c_{j,m} A~_{m,i} + M~_i) e^{i p_j theta_i}
//   kappa = sm_scale * log2(e), so scores come out in base-2 units for exp2.
//   This is the rebuilt-K score of the close reading §二.3 (RoPE after
//   reconstruction), reordered; no approximation.
// V is never rebuilt per token: the CTA accumulates sum_j p_j c_v,j in latent
// space and the combine pass applies W_up,v,t,h once.
#include <cmath>
#include <cstdio>

#include "lla_internal.cuh"

namespace lla {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide reductions for blockDim.x == 128 (4 warps); `red` holds 4 floats.
__device__ __forceinline__ float block_sum128(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  return red[0] + red[1] + red[2] + red[3];
}

__device__ __forceinline__ float block_max128(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  return fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
}

// ---------------------------------------------------------------- RoPE table

__global__ void rope_table_kernel(int max_pos, int half, double base, float2* table) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)max_pos * half) return;
  const int pos = (int)(idx / half);
  const int i = (int)(idx % half);
  const double theta = pow(base, -2.0 * i / (2.0 * half));
  double s, c;
  sincos((double)pos * theta, &s, &c);
  table[idx] = make_float2((float)c, (float)s);
}

// ---------------------------------------------------------------- packing

// W_up: per head [H][T][d][r] (LLA-2D [T][H][d][r]) -> [T][H][d][r], or with
// transpose != 0 -> [T][H][r][d] (the V up-projection, read column-wise).
__global__ void pack_wup_kernel(const float* __restrict__ in, float* __restrict__ out, int T,
                                int H, int d, int r, int per_head, int transpose) {
  const long long n = (long long)T * H * d * r;
  for (long long o = (long long)blockIdx.x * blockDim.x + threadIdx.x; o < n;
       o += (long long)gridDim.x * blockDim.x) {
    int m, i;
    long long rest;
    if (transpose) {
      i = (int)(o % d);
      rest = o / d;
      m = (int)(rest % r);
      rest /= r;
    } else {
      m = (int)(o % r);
      rest = o / r;
      i = (int)(rest % d);
      rest /= d;
    }
    const int h = (int)(rest % H);
    const int t = (int)(rest / H);
    const long long src = per_head ? ((((long long)h * T + t) * d + i) * r + m)
                                   : ((((long long)t * H + h) * d + i) * r + m);
    out[o] = in[src];
  }
}

// mu: per head [H][T*d] -> [T][H][d]; LLA-2D [T*H*d] is already (t, h, i).
__global__ void pack_mu_kernel(const float* __restrict__ in, float* __restrict__ out, int T, int H,
                               int d, int per_head) {
  const int n = T * H * d;
  for (int o = blockIdx.x * blockDim.x + threadIdx.x; o < n; o += gridDim.x * blockDim.x) {
    const int i = o % d;
    const int h = (o / d) % H;
    const int t = o / (d * H);
    out[o] = per_head ? in[(h * T + t) * d + i] : in[o];
  }
}

// W_down [L][W][r] fp32 -> [L][r][W] bf16 (round to nearest even).
__global__ void pack_wdown_kernel(const float* __restrict__ in, __nv_bfloat16* __restrict__ out,
                                  int L, int W, int r) {
  const long long n = (long long)L * W * r;
  for (long long o = (long long)blockIdx.x * blockDim.x + threadIdx.x; o < n;
       o += (long long)gridDim.x * blockDim.x) {
    const int k = (int)(o % W);
    const long long lm = o / W;
    const int m = (int)(lm % r);
    const int l = (int)(lm / r);
    out[o] = __float2bfloat16_rn(in[((long long)l * W + k) * r + m]);
  }
}

// bias[l][m] = sum_k mu_l[k] * W_bf16[l][m][k], accumulated in fp64.  One warp per (l, m).
__global__ void pack_bias_kernel(const float* __restrict__ mu, const __nv_bfloat16* __restrict__ wd,
                                 float* __restrict__ bias, int L, int W, int r) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= L * r) return;
  const int l = warp / r;
  const __nv_bfloat16* row = wd + (long long)warp * W;
  const float* m = mu + (long long)l * W;
  double acc = 0.0;
  for (int k = lane; k < W; k += 32) acc += (double)m[k] * (double)__bfloat162float(row[k]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) bias[warp] = (float)acc;
}

// Tensor-core encode operand images.  Chunk c of latent l is the [N][kc] tile of
// W_down^T (rows = latent index m, columns = input entries c*kc ...), rows >= r zero,
// stored the way a swizzled K-major TMA box lands in shared memory: the 16-byte
// unit u of row `row` (128-byte rows for kc = 64, 64-byte rows for kc = 32) sits at
// unit u ^ (row-group bits 7.. of its byte offset), so one bulk copy stages it.
__global__ void pack_wimg_kernel(const __nv_bfloat16* __restrict__ wd, __nv_bfloat16* __restrict__ img,
                                 int L, int W, int r, int N, int kc) {
  const int nch = W / kc;
  const long long total = (long long)L * nch * N * kc;
  const unsigned mask = kc == 64 ? 7u : 3u;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int col = (int)(e % kc);
    const int row = (int)((e / kc) % N);
    const long long tile = e / ((long long)kc * N);      // l * nch + c
    const int c = (int)(tile % nch);
    const int l = (int)(tile / nch);
    const __nv_bfloat16 v = row < r ? wd[((long long)l * r + row) * W + (long long)c * kc + col]
                                    : __float2bfloat16_rn(0.f);
    const unsigned o = (unsigned)(row * kc + col) * 2u;
    const unsigned so = o ^ (((o >> 7) & mask) << 4);
    img[tile * N * kc + so / 2] = v;
  }
}

// ---------------------------------------------------------------- encode

// One CTA per (token, latent l, K or V).  c[m] = sum_k x[k] W^T[m][k] - bias[m].
__global__ void __launch_bounds__(256) encode_kernel(
    const __nv_bfloat16* __restrict__ xk, const __nv_bfloat16* __restrict__ xv,
    const __nv_bfloat16* __restrict__ wdk, const __nv_bfloat16* __restrict__ wdv,
    const float* __restrict__ biask, const float* __restrict__ biasv, const int64_t* __restrict__ slot,
    int64_t n_slots, __nv_bfloat16* __restrict__ ck, __nv_bfloat16* __restrict__ cv,
    int32_t* status, int T, int H, int d, int r_k, int r_v, int per_head) {
  extern __shared__ float xs[];  // [W]
  const long long tok = blockIdx.x;
  const int l = blockIdx.y;
  const int kv = blockIdx.z;
  const int W = per_head ? T * d : T * H * d;
  const int L = per_head ? H : 1;
  const int64_t s = slot[tok];
  if (s < 0 || s >= n_slots) {
    if (threadIdx.x == 0 && l == 0 && kv == 0 && status) atomicOr(status, LLA_STATUS_SLOT_RANGE);
    return;
  }
  const __nv_bfloat16* x = (kv ? xv : xk) + tok * (long long)T * H * d;
  // Gather this latent's input row: per head the loop-major concat of head l.
  const int chunks = W / 8;
  for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
    const int k0 = c * 8;
    long long src;
    if (per_head) {
      const int t = k0 / d, i = k0 % d;
      src = ((long long)t * H + l) * d + i;
    } else {
      src = k0;
    }
    const uint4 raw = *reinterpret_cast<const uint4*>(x + src);
    const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(v2[e]);
      xs[k0 + 2 * e] = f.x;
      xs[k0 + 2 * e + 1] = f.y;
    }
  }
  __syncthreads();
  const int r = kv ? r_v : r_k;
  const __nv_bfloat16* wd = (kv ? wdv : wdk) + (long long)l * r * W;
  const float* bias = (kv ? biasv : biask) + (long long)l * r;
  __nv_bfloat16* dst = (kv ? cv : ck) + (long long)s * L * r + (long long)l * r;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int m = warp; m < r; m += blockDim.x >> 5) {
    const __nv_bfloat16* row = wd + (long long)m * W;
    float acc = 0.f;
    for (int k0 = lane * 8; k0 < W; k0 += 256) {
      const uint4 raw = *reinterpret_cast<const uint4*>(row + k0);
      const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(w2[e]);
        acc = fmaf(xs[k0 + 2 * e], f.x, acc);
        acc = fmaf(xs[k0 + 2 * e + 1], f.y, acc);
      }
    }
    acc = warp_sum(acc);
    if (lane == 0) dst[m] = __float2bfloat16_rn(acc - bias[m]);
  }
}

// ---------------------------------------------------------------- decode (CUDA cores)

constexpr int kPairChunk = 16;

// One CTA per (split, head, sequence); thread j of a tile owns history token j.
__global__ void __launch_bounds__(128) decode_partial_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int half = a.d >> 1;
  float2* At = reinterpret_cast<float2*>(smem_raw);                  // [r_k][half]
  float2* Mt = At + (size_t)a.r_k * half;                            // [half]
  float2* qc = Mt + half;                                            // [half]
  float* p_s = reinterpret_cast<float*>(qc + half);                  // [kTile]
  float* red = p_s + kTile;                                          // [8]
  __nv_bfloat16* cT = reinterpret_cast<__nv_bfloat16*>(red + 8);     // [r_k][kTile]

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;

  int n = a.ctx_len[b];
  if (n < 0 || n > a.n_cap) {
    if (tid == 0) atomicOr(a.status, LLA_STATUS_CTX_RANGE);
    n = n < 0 ? 0 : a.n_cap;
  }
  int qp = a.q_pos[b];
  if (qp < 0 || qp >= a.rope_max_pos) {
    if (tid == 0) atomicOr(a.status, LLA_STATUS_POSITION_RANGE);
    qp = 0;
  }

  // Rotated query as complex pairs.
  const float* qh = a.q + ((size_t)b * a.H + h) * a.d;
  for (int i = tid; i < half; i += blockDim.x) {
    const float2 e = a.rope[(size_t)qp * half + i];
    const float x0 = qh[i], x1 = qh[i + half];
    qc[i] = make_float2(x0 * e.x - x1 * e.y, x0 * e.y + x1 * e.x);
  }
  __syncthreads();
  // Query-absorbed up-projection A~ and bias M~.
  const float* W = a.wupk_t + (size_t)h * a.d * a.r_k;  // [d][r_k]
  const float* mu = a.muk_t + (size_t)h * a.d;
  for (int idx = tid; idx < a.r_k * half; idx += blockDim.x) {
    const int m = idx / half, i = idx % half;
    const float wr = W[(size_t)i * a.r_k + m], wi = W[(size_t)(i + half) * a.r_k + m];
    const float2 z = qc[i];
    At[idx] = make_float2(a.kappa * (z.x * wr + z.y * wi), a.kappa * (z.x * wi - z.y * wr));
  }
  for (int i = tid; i < half; i += blockDim.x) {
    const float2 z = qc[i];
    const float mr = mu[i], mi = mu[i + half];
    Mt[i] = make_float2(a.kappa * (z.x * mr + z.y * mi), a.kappa * (z.x * mi - z.y * mr));
  }

  const int tok_begin = split * a.tiles_per_split * kTile;
  int tok_end = tok_begin + a.tiles_per_split * kTile;
  if (tok_end > n) tok_end = n;

  float m_run = -INFINITY, l_run = 0.f;
  float o0 = 0.f, o1 = 0.f;  // latent dims 2*tid, 2*tid+1
  const bool own_v = 2 * tid < a.r_v;
  const size_t seq_k = (size_t)b * a.n_cap * a.lat_tok_k + (size_t)h * a.lat_head_k;
  const size_t seq_v = (size_t)b * a.n_cap * a.lat_tok_v + (size_t)h * a.lat_head_v;
  const int32_t* pos_b = a.positions + (size_t)b * a.n_cap;

  for (int t0 = tok_begin; t0 < tok_end; t0 += kTile) {
    const int cnt = min(kTile, tok_end - t0);
    __syncthreads();
    // Stage the K latent tile transposed: cT[m][j].
    const int cpr = a.r_k / 8;
    for (int idx = tid; idx < kTile * cpr; idx += blockDim.x) {
      const int j = idx / cpr, c = idx % cpr;
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (j < cnt)
        raw = *reinterpret_cast<const uint4*>(a.ck + seq_k + (size_t)(t0 + j) * a.lat_tok_k + c * 8);
      const __nv_bfloat16* v = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
      for (int e = 0; e < 8; ++e) cT[(size_t)(c * 8 + e) * kTile + j] = v[e];
    }
    __syncthreads();

    float s = -INFINITY;
    if (tid < cnt) {
      int p = pos_b[t0 + tid];
      if (p < 0 || p >= a.rope_max_pos) {
        atomicOr(a.status, LLA_STATUS_POSITION_RANGE);
        p = 0;
      }
      const float2* E = a.rope + (size_t)p * half;
      float acc_s = 0.f;
      for (int p0 = 0; p0 < half; p0 += kPairChunk) {
        float ur[kPairChunk], ui[kPairChunk];
#pragma unroll
        for (int q = 0; q < kPairChunk; ++q) {
          const float2 z = Mt[p0 + q];
          ur[q] = z.x;
          ui[q] = z.y;
        }
        for (int m = 0; m < a.r_k; ++m) {
          const float c = __bfloat162float(cT[(size_t)m * kTile + tid]);
          const float4* row = reinterpret_cast<const float4*>(At + (size_t)m * half + p0);
#pragma unroll
          for (int q = 0; q < kPairChunk / 2; ++q) {
            const float4 w = row[q];
            ur[2 * q] = fmaf(c, w.x, ur[2 * q]);
            ui[2 * q] = fmaf(c, w.y, ui[2 * q]);
            ur[2 * q + 1] = fmaf(c, w.z, ur[2 * q + 1]);
            ui[2 * q + 1] = fmaf(c, w.w, ui[2 * q + 1]);
          }
        }
#pragma unroll
        for (int q = 0; q < kPairChunk; ++q) {
          const float2 e = E[p0 + q];
          acc_s = fmaf(ur[q], e.x, acc_s);
          acc_s = fmaf(-ui[q], e.y, acc_s);
        }
      }
      s = acc_s;
    }
    // Online softmax over this tile (base 2).
    const float m_tile = block_max128(s, red);
    const float m_new = fmaxf(m_run, m_tile);
    const float alpha = (m_run == -INFINITY) ? 0.f : exp2f(m_run - m_new);
    const float pj = (tid < cnt) ? exp2f(s - m_new) : 0.f;
    p_s[tid] = pj;
    const float l_tile = block_sum128(pj, red + 4);
    l_run = l_run * alpha + l_tile;
    m_run = m_new;
    // Latent-space V accumulation; p_s is visible after the reduction's barriers.
    o0 *= alpha;
    o1 *= alpha;
    if (own_v) {
      const __nv_bfloat16* vb = a.cv + seq_v + (size_t)t0 * a.lat_tok_v + 2 * tid;
      for (int j = 0; j < cnt; ++j) {
        const float2 v = __bfloat1622float2(
            *reinterpret_cast<const __nv_bfloat162*>(vb + (size_t)j * a.lat_tok_v));
        const float pw = p_s[j];
        o0 = fmaf(pw, v.x, o0);
        o1 = fmaf(pw, v.y, o1);
      }
    }
  }

  float* part = a.partials + (((size_t)b * a.H + h) * a.S + split) * (2 + a.r_v);
  if (tid == 0) {
    part[0] = m_run;
    part[1] = l_run;
  }
  if (own_v) {
    part[2 + 2 * tid] = o0;
    part[3 + 2 * tid] = o1;
  }
}

// Merge the splits, add the in-flight token and up-project V once.
// Grid (H, B, ceil(d / 32)); 512 threads.  Block z computes output rows
// [32 z, 32 z + 32) of (b, h); every phase issues all of its global loads at once.
constexpr int kCombineThreads = 512;

__global__ void __launch_bounds__(kCombineThreads) decode_combine_kernel(DecodeArgs a) {
  __shared__ float olat[256];
  __shared__ float mw[kMaxSplits];
  __shared__ float red[16];
  __shared__ float seg[16][33];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const size_t bh = (size_t)b * a.H + h;
  const float* parts = a.partials + bh * a.S * (2 + a.r_v);
  // split maxima, and the in-flight token's score
  // (same position for query and key: their relative rotation is the identity)
  float m_s = -INFINITY, dot = 0.f;
  if (tid < a.S) m_s = parts[(size_t)tid * (2 + a.r_v)];
  if (tid < a.d) dot = a.q[bh * a.d + tid] * a.k_self[bh * a.d + tid];
  const float mx = warp_max(m_s), dsum = warp_sum(dot);
  if (lane == 0) {
    red[warp] = mx;
    seg[warp][32] = dsum;
  }
  __syncthreads();
  float M_hist = red[0], s_self = 0.f;
  for (int w = 1; w < 16; ++w) M_hist = fmaxf(M_hist, red[w]);
  for (int w = 0; w < 16; ++w) s_self += seg[w][32];
  s_self *= a.kappa;
  const float M = fmaxf(M_hist, s_self);
  const float wgt = tid < a.S ? exp2f(m_s - M) : 0.f;
  if (tid < a.S) mw[tid] = wgt;
  __syncthreads();
  float l_hist = 0.f;
  for (int s = 0; s < a.S; ++s) l_hist = fmaf(parts[(size_t)s * (2 + a.r_v) + 1], mw[s], l_hist);
  const float w_self = exp2f(s_self - M);
  const float inv = 1.f / (l_hist + w_self);
  for (int m = tid; m < a.r_v; m += kCombineThreads) {
    float acc = 0.f;
    for (int s = 0; s < a.S; ++s) acc = fmaf(parts[(size_t)s * (2 + a.r_v) + 2 + m], mw[s], acc);
    olat[m] = acc * inv;
  }
  __syncthreads();
  // W_up,v,t,h is packed transposed ([r_v][d]); warp w sums latent dims m = w, w + 16, ...
  // for the 32 rows i of this block (lane = row), all loads independent.
  const int i = blockIdx.z * 32 + lane;
  const float* Wt = a.wupv_t + (size_t)h * a.d * a.r_v;
  float acc = 0.f;
  if (i < a.d) {
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int m = warp + 16 * k;
      if (m < a.r_v) acc = fmaf(Wt[(size_t)m * a.d + i], olat[m], acc);
    }
  }
  seg[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && i < a.d) {
    float y = 0.f;
#pragma unroll
    for (int w = 0; w < 16; ++w) y += seg[w][lane];
    const float* muv = a.muv_t + (size_t)h * a.d;
    a.out[bh * a.d + i] = y + (l_hist * inv) * muv[i] + (w_self * inv) * a.v_self[bh * a.d + i];
  }
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && tid == 0) {
    a.status[1] = a.status[0];
    a.status[0] = 0;
  }
}

size_t decode_partial_smem(const DecodeArgs& a) {
  const int half = a.d / 2;
  return (size_t)a.r_k * half * sizeof(float2) + 2 * half * sizeof(float2) +
         (kTile + 8) * sizeof(float) + (size_t)a.r_k * kTile * sizeof(__nv_bfloat16);
}

}  // namespace

cudaError_t launch_rope_table(const lla_cfg& c, int max_pos, float2* table, cudaStream_t s) {
  const int half = rotary_dims(c) / 2;
  const long long n = (long long)max_pos * half;
  const int threads = 256;
  const long long blocks = (n + threads - 1) / threads;
  rope_table_kernel<<<(unsigned)blocks, threads, 0, s>>>(max_pos, half, (double)c.rope_base, table);
  return cudaGetLastError();
}

cudaError_t launch_pack(const lla_cfg& c, const PackedLayout& L, const float* wdk,
                        const float* wdv, const float* wupk, const float* wupv,
                        const float* muk, const float* muv, char* packed, cudaStream_t s) {
  const int per_head = c.mode == LLA_MODE_PER_HEAD;
  const int T = c.T, H = c.H, d = c.d_head;
  pack_wup_kernel<<<512, 256, 0, s>>>(wupk, reinterpret_cast<float*>(packed + L.wupk), T, H, d,
                                      c.r_k, per_head, 0);
  pack_wup_kernel<<<512, 256, 0, s>>>(wupv, reinterpret_cast<float*>(packed + L.wupv), T, H, d,
                                      c.r_v, per_head, 1);
  pack_mu_kernel<<<64, 256, 0, s>>>(muk, reinterpret_cast<float*>(packed + L.muk), T, H, d, per_head);
  pack_mu_kernel<<<64, 256, 0, s>>>(muv, reinterpret_cast<float*>(packed + L.muv), T, H, d, per_head);
  auto* wdk_bf = reinterpret_cast<__nv_bfloat16*>(packed + L.wdk);
  auto* wdv_bf = reinterpret_cast<__nv_bfloat16*>(packed + L.wdv);
  pack_wdown_kernel<<<512, 256, 0, s>>>(wdk, wdk_bf, L.L, L.W, c.r_k);
  pack_wdown_kernel<<<512, 256, 0, s>>>(wdv, wdv_bf, L.L, L.W, c.r_v);
  // mu in the input layout is already the concatenated mean per latent ([L][W]).
  const int kc = encode_kc(c);
  pack_wimg_kernel<<<512, 256, 0, s>>>(wdk_bf, reinterpret_cast<__nv_bfloat16*>(packed + L.wimgk),
                                       L.L, L.W, c.r_k, pad16(c.r_k), kc);
  pack_wimg_kernel<<<512, 256, 0, s>>>(wdv_bf, reinterpret_cast<__nv_bfloat16*>(packed + L.wimgv),
                                       L.L, L.W, c.r_v, pad16(c.r_v), kc);
  const int wk = L.L * c.r_k, wv = L.L * c.r_v;
  pack_bias_kernel<<<(wk * 32 + 255) / 256, 256, 0, s>>>(
      muk, wdk_bf, reinterpret_cast<float*>(packed + L.biask), L.L, L.W, c.r_k);
  pack_bias_kernel<<<(wv * 32 + 255) / 256, 256, 0, s>>>(
      muv, wdv_bf, reinterpret_cast<float*>(packed + L.biasv), L.L, L.W, c.r_v);
  return cudaGetLastError();
}

cudaError_t launch_encode(const lla_cfg& c, const PackedLayout& L, const char* packed,
                          int64_t n_tok, const __nv_bfloat16* xk, const __nv_bfloat16* xv,
                          const int64_t* slot, int64_t n_slots, __nv_bfloat16* ck,
                          __nv_bfloat16* cv, int32_t* status, cudaStream_t s) {
  const size_t smem = (size_t)L.W * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(encode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)n_tok, (unsigned)L.L, 2);
  encode_kernel<<<grid, 256, smem, s>>>(
      xk, xv, reinterpret_cast<const __nv_bfloat16*>(packed + L.wdk),
      reinterpret_cast<const __nv_bfloat16*>(packed + L.wdv),
      reinterpret_cast<const float*>(packed + L.biask),
      reinterpret_cast<const float*>(packed + L.biasv), slot, n_slots, ck, cv, status, c.T, c.H,
      c.d_head, c.r_k, c.r_v, c.mode == LLA_MODE_PER_HEAD);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s, int* launches) {
  *launches = 0;
  if (a.S > 0) {
    const size_t smem = decode_partial_smem(a);
    cudaError_t e = cudaFuncSetAttribute(decode_partial_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)a.S, (unsigned)a.H, (unsigned)a.B);
    decode_partial_kernel<<<grid, kTile, smem, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  cudaError_t e = launch_combine(a, s);
  if (e == cudaSuccess) ++*launches;
  return e;
}

cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t s) {
  dim3 g2((unsigned)a.H, (unsigned)a.B, (unsigned)((a.d + 31) / 32));
  decode_combine_kernel<<<g2, kCombineThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace lla
