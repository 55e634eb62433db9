// Bandwidth- and latency-bound kernels of the denoising pass: embedding gather,
// RMSNorm, MoE router / top-k / permute / gather / combine, the LM-head partial merge,
// and the commit (sampler) kernel.
#pragma once

#include "common.cuh"

namespace dllm {

// ---------------------------------------------------------------- a1: embedding

// x[t] = Emb[token] as fp32; a masked canvas position reads the [MASK] row.
__global__ void embed_kernel(const bf16_t* __restrict__ emb, const int32_t* __restrict__ tokens,
                             const uint8_t* __restrict__ mask, int mask_id, int d, float* __restrict__ x) {
  pdl_begin();
  const int t = blockIdx.x;
  int tok = tokens[t];
  if (mask != nullptr && mask[t]) tok = mask_id;
  const uint4* src = reinterpret_cast<const uint4*>(emb + (long)tok * d);
  float4* dst = reinterpret_cast<float4*>(x + (long)t * d);
  for (int c = threadIdx.x; c < d / 8; c += blockDim.x) {
    uint4 v = src[c];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
    dst[2 * c] = make_float4(f[0], f[1], f[2], f[3]);
    dst[2 * c + 1] = make_float4(f[4], f[5], f[6], f[7]);
  }
}

// ---------------------------------------------------------------- a2/a6/a12: RMSNorm

// Writes v as bf16 terms: y = bf16(v), y_lo = bf16(v - y) and, when y_lo2 is given, the
// third term y_lo2 = bf16(v - y - y_lo), so that y + y_lo + y_lo2 carries all of v's fp32
// bits (the QKV projection's operand; the other GEMMs read the (y, y_lo) pair).
DLLM_DEV void store_norm_terms(bf16_t* y, bf16_t* y_lo, bf16_t* y_lo2, long t, int d, int c, float4 v) {
  uint32_t h0, l0, h1, l1;
  if (y_lo2) {
    uint32_t m0, m1;
    split3_bf16x2(v.x, v.y, h0, m0, l0);
    split3_bf16x2(v.z, v.w, h1, m1, l1);
    reinterpret_cast<uint2*>(y + t * d)[c] = make_uint2(h0, h1);
    reinterpret_cast<uint2*>(y_lo + t * d)[c] = make_uint2(m0, m1);
    reinterpret_cast<uint2*>(y_lo2 + t * d)[c] = make_uint2(l0, l1);
    return;
  }
  split_bf16x2(v.x, v.y, h0, l0);
  split_bf16x2(v.z, v.w, h1, l1);
  reinterpret_cast<uint2*>(y + t * d)[c] = make_uint2(h0, h1);
  reinterpret_cast<uint2*>(y_lo + t * d)[c] = make_uint2(l0, l1);
}

// v = x * rsqrt(mean(x^2) + eps) * g, written as bf16 terms (store_norm_terms); rstd[t]
// kept for the fp32 router.
//
// With nparts > 0 the row first takes the split-K partial sums of the GEMM before it:
// x[t] += part[0][t] + part[1][t] + ... (slice order, partial s at part + s * pstride),
// written back to x, and the norm is taken of the updated row.
__global__ void rmsnorm_kernel(float* __restrict__ x, const float* __restrict__ part, int nparts, long pstride,
                               const float* __restrict__ g, int d, float eps,
                               bf16_t* __restrict__ y, bf16_t* __restrict__ y_lo, bf16_t* __restrict__ y_lo2,
                               float* __restrict__ rstd) {
  pdl_begin();
  const int t = blockIdx.x;
  float4* xr = reinterpret_cast<float4*>(x + (long)t * d);
  float ss = 0.f;
  for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
    float4 v = xr[c];
    if (nparts > 0) {
      const float4* pr = reinterpret_cast<const float4*>(part + (long)t * d) + c;
      // four partials' loads at a time, all in flight before they are added (in slice order)
      for (int s0 = 0; s0 < nparts; s0 += 4) {
        float4 a[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) a[u] = s0 + u < nparts ? pr[(s0 + u) * (pstride / 4)] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (s0 + u < nparts) {
            v.x += a[u].x;
            v.y += a[u].y;
            v.z += a[u].z;
            v.w += a[u].w;
          }
        }
      }
      xr[c] = v;
    }
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  __shared__ float red[32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float r = rsqrtf(red[0] / (float)d + eps);
  if (threadIdx.x == 0 && rstd != nullptr) rstd[t] = r;
  const float4* gr = reinterpret_cast<const float4*>(g);
  for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
    const float4 v = xr[c], gg = gr[c];   // with partials: this thread's own writes above
    store_norm_terms(y, y_lo, y_lo2, t, d, c, make_float4(v.x * r * gg.x, v.y * r * gg.y, v.z * r * gg.z, v.w * r * gg.w));
  }
}

// ---------------------------------------------------------------- a7: router + top-k

// logits[t][e] = sum_k (x[t][k] * rstd[t] * g[k]) * Wr[e][k], all in fp32.
// Block (blockIdx.x, blockIdx.y) = (kRouterTok tokens, kRouterExp experts): the tokens'
// normalised rows sit in shared memory; each of the 8 warps owns kRouterExp / 8 experts,
// its lanes split the d-long dot products in 8-element chunks, and the chunk loop is
// unrolled (d <= kRouterMaxChunks * 256) so that all of a warp's weight loads are in
// flight together instead of one dependent load per iteration.
constexpr int kRouterTok = 4;
constexpr int kRouterExp = 32;
constexpr int kRouterMaxChunks = 16;   // d <= 4096
__global__ void __launch_bounds__(256) router_kernel(const float* __restrict__ x, const float* __restrict__ rstd,
                                                     const float* __restrict__ g, const bf16_t* __restrict__ wr,
                                                     int T, int d, int E, float* __restrict__ logits) {
  pdl_begin();
  extern __shared__ float xs[];   // [kRouterTok][d]
  const int t0 = blockIdx.x * kRouterTok;
  for (int i = threadIdx.x; i < kRouterTok * d / 4; i += blockDim.x) {
    const int tk = (4 * i) / d, k = (4 * i) % d;
    const int t = t0 + tk;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t < T) {
      const float r = rstd[t];
      const float4 xv = *reinterpret_cast<const float4*>(x + (long)t * d + k);
      const float4 gv = *reinterpret_cast<const float4*>(g + k);
      v = make_float4(xv.x * r * gv.x, xv.y * r * gv.y, xv.z * r * gv.z, xv.w * r * gv.w);
    }
    reinterpret_cast<float4*>(xs)[i] = v;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int EPW = kRouterExp / 8;   // experts per warp
  const int e0 = blockIdx.y * kRouterExp + warp * EPW;
  const int nchunks = d / 256;
  float acc[EPW][kRouterTok];
#pragma unroll
  for (int j = 0; j < EPW; ++j)
#pragma unroll
    for (int tk = 0; tk < kRouterTok; ++tk) acc[j][tk] = 0.f;
#pragma unroll
  for (int c = 0; c < kRouterMaxChunks; ++c) {
    if (c < nchunks) {
      const int k = c * 256 + lane * 8;
      uint4 wv[EPW];
#pragma unroll
      for (int j = 0; j < EPW; ++j) {
        const int e = e0 + j;
        wv[j] = e < E ? *reinterpret_cast<const uint4*>(wr + (long)e * d + k) : make_uint4(0, 0, 0, 0);
      }
      float xf[kRouterTok][8];
#pragma unroll
      for (int tk = 0; tk < kRouterTok; ++tk) {
        const float4 a = *reinterpret_cast<const float4*>(xs + tk * d + k);
        const float4 b = *reinterpret_cast<const float4*>(xs + tk * d + k + 4);
        xf[tk][0] = a.x; xf[tk][1] = a.y; xf[tk][2] = a.z; xf[tk][3] = a.w;
        xf[tk][4] = b.x; xf[tk][5] = b.y; xf[tk][6] = b.z; xf[tk][7] = b.w;
      }
#pragma unroll
      for (int j = 0; j < EPW; ++j) {
        const uint32_t ww[4] = {wv[j].x, wv[j].y, wv[j].z, wv[j].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float w0 = __uint_as_float(ww[i] << 16), w1 = __uint_as_float(ww[i] & 0xFFFF0000u);
#pragma unroll
          for (int tk = 0; tk < kRouterTok; ++tk) {
            acc[j][tk] = fmaf(w0, xf[tk][2 * i], acc[j][tk]);
            acc[j][tk] = fmaf(w1, xf[tk][2 * i + 1], acc[j][tk]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < EPW; ++j)
#pragma unroll
    for (int tk = 0; tk < kRouterTok; ++tk) {
      const float s = warp_sum(acc[j][tk]);
      if (lane == 0 && t0 + tk < T && e0 + j < E) logits[(long)(t0 + tk) * E + e0 + j] = s;
    }
}

// Top-k of token t's E logits (ties to the lower expert) and the softmax of the k
// selected logits as gates, by one warp (E <= 256, k <= 32). A NaN logit counts as -inf,
// so every selected index is a valid expert whatever the hidden state holds.
DLLM_DEV void topk_token(const float* logits, int t, int E, int k, int32_t* idx, float* gate, int lane) {
  float v[8];
  bool taken[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    const float x = (e < E) ? logits[(long)t * E + e] : -INFINITY;
    v[j] = x != x ? -INFINITY : x;
    taken[j] = (e >= E);
  }
  float sel_v = 0.f, top = 0.f;
  int sel_i = 0;
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      if (!taken[j] && (v[j] > bv || (v[j] == bv && e < bi))) { bv = v[j]; bi = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (lane + 32 * j == bi) taken[j] = true;
    if (r == 0) top = bv;
    if (lane == r) { sel_v = bv; sel_i = bi; }
  }
  const float ex = (lane < k) ? expf(sel_v - top) : 0.f;
  const float z = warp_sum(ex);
  if (lane < k) {
    idx[(long)t * k + lane] = sel_i;
    gate[(long)t * k + lane] = ex / z;
  }
}

// With nparts > 0 the router GEMM left split-K partial sums (partial s at
// part + s * pstride): each lane first adds, in slice order, the partials of the logits it
// reads and stores them in `logits` (the full logits stay available to the debug copies).
__global__ void topk_kernel(float* __restrict__ logits, int T, int E, int k, int32_t* __restrict__ idx,
                            float* __restrict__ gate, const float* __restrict__ part, int nparts, long pstride) {
  pdl_begin();
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  if (nparts > 0) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = 0.f;
    // four partials' loads at a time, all in flight before they are added (in slice order)
    for (int s0 = 0; s0 < nparts; s0 += 4) {
      float pv[4][8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float* ps = part + (s0 + u) * pstride + (long)t * E;
#pragma unroll
        for (int j = 0; j < 8; ++j) pv[u][j] = (s0 + u < nparts && lane + 32 * j < E) ? ps[lane + 32 * j] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (s0 + u < nparts) v[j] += pv[u][j];
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (lane + 32 * j < E) logits[(long)t * E + lane + 32 * j] = v[j];
  }
  topk_token(logits, t, E, k, idx, gate, lane);
}

// Debug: replace the top-k experts with given ones (the oracle's), gates recomputed
// from this pass's own logits at those experts. One thread per token.
__global__ void force_route_kernel(const float* __restrict__ logits, const int32_t* __restrict__ forced, int T,
                                   int E, int k, int32_t* __restrict__ idx, float* __restrict__ gate) {
  pdl_begin();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  float mx = -INFINITY;
  for (int j = 0; j < k; ++j) mx = fmaxf(mx, logits[(long)t * E + forced[(long)t * k + j]]);
  float z = 0.f;
  for (int j = 0; j < k; ++j) z += expf(logits[(long)t * E + forced[(long)t * k + j]] - mx);
  for (int j = 0; j < k; ++j) {
    const int e = forced[(long)t * k + j];
    idx[(long)t * k + j] = e;
    gate[(long)t * k + j] = expf(logits[(long)t * E + e] - mx) / z;
  }
}

// Dense FFN as one expert with gate 1.
__global__ void dense_route_kernel(int T, int32_t* idx, float* gate) {
  pdl_begin();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < T) { idx[t] = 0; gate[t] = 1.f; }
}

// ---------------------------------------------------------------- a8: permute

// Counting sort of the N = T*k assignments by expert (one CTA of 1024 threads).
// offsets[E+1]: expert ranges in the sorted order; slot_of[i]: sorted position of
// assignment i = t*k + j; row_token[slot]: its token. Within an expert, slots are handed
// out by an atomic cursor; no value depends on that order (each token's column of an
// expert GEMM is computed on its own and the combine sums in the fixed j order).
// Also lists the experts with at least one assignment (routed[0..n_routed), ascending)
// with the prefix sums of their chunk counts ceil(count / bn) for the persistent grouped
// GEMMs, and stores n_routed in *routed_stat when given. E <= 256.
__global__ void __launch_bounds__(1024) permute_kernel(const int32_t* __restrict__ idx, int N, int k, int E,
                                                       int32_t* __restrict__ offsets, int32_t* __restrict__ slot_of,
                                                       int32_t* __restrict__ row_token, int32_t* __restrict__ routed,
                                                       int32_t* __restrict__ n_routed, int32_t* __restrict__ chunk_prefix,
                                                       int bn, int32_t* __restrict__ routed_stat) {
  pdl_begin();
  __shared__ int cnt[256];
  __shared__ int cur[256];
  const int tid = threadIdx.x, lane = tid & 31;
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int i = tid; i < N; i += blockDim.x) atomicAdd(&cnt[idx[i]], 1);
  __syncthreads();
  if (tid < 32) {
    // lane owns experts [lane * per, lane * per + per); exclusive scans of the counts,
    // of the routed flags and of the chunk counts
    const int per = (E + 31) / 32;
    int c_sum = 0, r_sum = 0, ch_sum = 0;
    for (int q = 0; q < per; ++q) {
      const int e = lane * per + q;
      const int c = e < E ? cnt[e] : 0;
      c_sum += c;
      r_sum += c > 0;
      ch_sum += (c + bn - 1) / bn;
    }
    int c_pre = c_sum, r_pre = r_sum, ch_pre = ch_sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, c_pre, o);
      const int b = __shfl_up_sync(0xffffffffu, r_pre, o);
      const int d = __shfl_up_sync(0xffffffffu, ch_pre, o);
      if (lane >= o) {
        c_pre += a;
        r_pre += b;
        ch_pre += d;
      }
    }
    c_pre -= c_sum;
    r_pre -= r_sum;
    ch_pre -= ch_sum;
    for (int q = 0; q < per; ++q) {
      const int e = lane * per + q;
      if (e >= E) break;
      const int c = cnt[e];
      offsets[e] = c_pre;
      cur[e] = c_pre;
      if (c > 0) {
        routed[r_pre] = e;
        chunk_prefix[r_pre] = ch_pre;
        ++r_pre;
        ch_pre += (c + bn - 1) / bn;
      }
      c_pre += c;
    }
    if (lane == 31) {
      offsets[E] = c_pre;
      chunk_prefix[r_pre] = ch_pre;
      *n_routed = r_pre;
      if (routed_stat) *routed_stat = r_pre;
    }
  }
  __syncthreads();
  for (int i = tid; i < N; i += blockDim.x) {
    const int s = atomicAdd(&cur[idx[i]], 1);
    slot_of[i] = s;
    row_token[s] = i / k;
  }
}

// xg[slot] = y[row_token[slot]] for the hi and lo bf16 rows: the B operand pair of the
// grouped gate/up GEMM.
__global__ void gather_rows_kernel(const bf16_t* __restrict__ y, const bf16_t* __restrict__ y_lo,
                                   const int32_t* __restrict__ row_token, int N, int d, bf16_t* __restrict__ xg,
                                   bf16_t* __restrict__ xg_lo) {
  pdl_begin();
  const int s = blockIdx.x;
  if (s >= N) return;
  const long src_row = (long)row_token[s] * d;
  const uint4* src = reinterpret_cast<const uint4*>(y + src_row);
  const uint4* src_lo = reinterpret_cast<const uint4*>(y_lo + src_row);
  uint4* dst = reinterpret_cast<uint4*>(xg + (long)s * d);
  uint4* dst_lo = reinterpret_cast<uint4*>(xg_lo + (long)s * d);
  for (int c = threadIdx.x; c < d / 8; c += blockDim.x) {
    dst[c] = src[c];
    dst_lo[c] = src_lo[c];
  }
}

// ---------------------------------------------------------------- a11: combine

// x[t] += sum_j gate[t][j] * o[slot_of[t*k + j]], j in fixed order 0..k-1.
// Token t's routed rows and gates, held in registers (k <= kMaxK), so that the k row
// loads of one column chunk are all in flight together.
constexpr int kMaxK = 8;
struct CombineRow {
  const float4* row[kMaxK];
  float w[kMaxK];
  int k;
  DLLM_DEV CombineRow(const float* o, const int32_t* slot_of, const float* gate, int t, int k_, int d) : k(k_) {
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      const bool on = j < k;
      row[j] = reinterpret_cast<const float4*>(o + (long)(on ? slot_of[(long)t * k + j] : 0) * d);
      w[j] = on ? gate[(long)t * k + j] : 0.f;
    }
  }
  // sum_j w_j * o[slot_j][4c .. 4c+3], accumulated in j order
  DLLM_DEV float4 at(int c) const {
    float4 v[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) v[j] = j < k ? row[j][c] : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k) {
        acc.x = fmaf(w[j], v[j].x, acc.x);
        acc.y = fmaf(w[j], v[j].y, acc.y);
        acc.z = fmaf(w[j], v[j].z, acc.z);
        acc.w = fmaf(w[j], v[j].w, acc.w);
      }
    }
    return acc;
  }
};

__global__ void combine_kernel(float* __restrict__ x, const float* __restrict__ o, const int32_t* __restrict__ slot_of,
                               const float* __restrict__ gate, int k, int d) {
  pdl_begin();
  const int t = blockIdx.x;
  float4* xr = reinterpret_cast<float4*>(x + (long)t * d);
  const CombineRow cr(o, slot_of, gate, t, k, d);
  for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
    const float4 acc = cr.at(c);
    float4 xv = xr[c];
    xv.x += acc.x;
    xv.y += acc.y;
    xv.z += acc.z;
    xv.w += acc.w;
    xr[c] = xv;
  }
}

// combine_kernel followed by the RMSNorm that comes next (the next layer's attention
// norm, or the final norm before the LM head): x is updated in place, then
// v = x * rsqrt(mean(x^2) + eps) * g is written as the (hi, lo) bf16 pair. One block per
// token; the same per-row arithmetic as combine_kernel and rmsnorm_kernel.
constexpr int kCombineChunks = 3;   // float4 columns per thread: d / 4 <= 3 * blockDim

// Two 256-thread blocks per SM (at most 128 registers a thread): all 256 tokens of a canvas
// stay resident with their loads in flight (measured 0.31 vs 0.36 ms per 26B canvas pass
// with one block per SM, 0.47 before the loads were issued together).
__global__ void __launch_bounds__(256, 2) combine_norm_kernel(float* __restrict__ x, const float* __restrict__ o,
                                                           const int32_t* __restrict__ slot_of,
                                                           const float* __restrict__ gate, int k, int d,
                                                           const float* __restrict__ g, float eps,
                                                           bf16_t* __restrict__ y, bf16_t* __restrict__ y_lo,
                                                           bf16_t* __restrict__ y_lo2) {
  pdl_begin();
  const int t = blockIdx.x;
  float4* xr = reinterpret_cast<float4*>(x + (long)t * d);
  const float4* gr = reinterpret_cast<const float4*>(g);
  const int n4 = d / 4;
  const CombineRow cr(o, slot_of, gate, t, k, d);
  // every load of this thread's first kCombineChunks float4 columns is issued before any
  // is used: the k routed rows, x and the gains (a 256-thread block covers d <= 3072 this
  // way; wider rows finish column by column below)
  float4 v[kCombineChunks][kMaxK], xv[kCombineChunks], gv[kCombineChunks];
#pragma unroll
  for (int i = 0; i < kCombineChunks; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    const bool on = c < n4;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) v[i][j] = (on && j < k) ? cr.row[j][c] : make_float4(0.f, 0.f, 0.f, 0.f);
    xv[i] = on ? xr[c] : make_float4(0.f, 0.f, 0.f, 0.f);
    gv[i] = on ? gr[c] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kCombineChunks; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    if (c >= n4) continue;
    // the same per-column arithmetic as combine_kernel: sum_j w_j o_j in j order, then + x
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k) {
        acc.x = fmaf(cr.w[j], v[i][j].x, acc.x);
        acc.y = fmaf(cr.w[j], v[i][j].y, acc.y);
        acc.z = fmaf(cr.w[j], v[i][j].z, acc.z);
        acc.w = fmaf(cr.w[j], v[i][j].w, acc.w);
      }
    }
    xv[i].x += acc.x;
    xv[i].y += acc.y;
    xv[i].z += acc.z;
    xv[i].w += acc.w;
    xr[c] = xv[i];
    ss += xv[i].x * xv[i].x + xv[i].y * xv[i].y + xv[i].z * xv[i].z + xv[i].w * xv[i].w;
  }
  // rows wider than kCombineChunks * blockDim float4s: the rest column by column
  for (int c = threadIdx.x + kCombineChunks * blockDim.x; c < n4; c += blockDim.x) {
    const float4 acc = cr.at(c);
    float4 a = xr[c];
    a.x += acc.x;
    a.y += acc.y;
    a.z += acc.z;
    a.w += acc.w;
    xr[c] = a;
    ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
  }
  __shared__ float red[32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float a = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    a = warp_sum(a);
    if (threadIdx.x == 0) red[0] = a;
  }
  __syncthreads();
  const float r = rsqrtf(red[0] / (float)d + eps);
#pragma unroll
  for (int i = 0; i < kCombineChunks; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    if (c >= n4) continue;
    store_norm_terms(y, y_lo, y_lo2, t, d, c,
                     make_float4(xv[i].x * r * gv[i].x, xv[i].y * r * gv[i].y, xv[i].z * r * gv[i].z,
                                 xv[i].w * r * gv[i].w));
  }
  for (int c = threadIdx.x + kCombineChunks * blockDim.x; c < n4; c += blockDim.x) {
    const float4 a = xr[c], gg = gr[c];   // this thread's own writes above
    store_norm_terms(y, y_lo, y_lo2, t, d, c, make_float4(a.x * r * gg.x, a.y * r * gg.y, a.z * r * gg.z, a.w * r * gg.w));
  }
}

// ---------------------------------------------------------------- a13: LM-head merge

DLLM_DEV void lse_combine(float& m, float& s, int& i, float m2, float s2, int i2) {
  constexpr float kLog2e = 1.4426950408889634f;
  if (m2 > m) {
    s = s2 + s * exp2f((m - m2) * kLog2e);
    m = m2;
    i = i2;
  } else if (m2 < m) {
    s += s2 * exp2f((m2 - m) * kLog2e);
  } else {
    s += s2;
    i = min(i, i2);
  }
}

// conf[t] = 1 / sum_v exp(l_v - max), argmax[t] = lowest id reaching the max.
// One warp per row over the row's vocabulary-tile partials. If a kernel before this one
// gave up a bounded wait (*err != 0), the partials are incomplete: every row gets
// conf = NaN and argmax = -1 instead.
__global__ void lm_merge_kernel(const float* __restrict__ pm, const float* __restrict__ ps,
                                const int32_t* __restrict__ pi, int rows, int n_tiles, float* __restrict__ conf,
                                int32_t* __restrict__ argmax, const int* __restrict__ err) {
  pdl_begin();
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= rows) return;
  if (err && *err) {
    if (lane == 0) {
      conf[t] = __int_as_float(0x7fc00000);
      argmax[t] = -1;
    }
    return;
  }
  float m = -INFINITY, s = 0.f;
  int i = 0x7fffffff;
  for (int j = lane; j < n_tiles; j += 32) {
    const long o = (long)t * n_tiles + j;
    lse_combine(m, s, i, pm[o], ps[o], pi[o]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, off);
    const int i2 = __shfl_xor_sync(0xffffffffu, i, off);
    lse_combine(m, s, i, m2, s2, i2);
  }
  if (lane == 0) {
    conf[t] = 1.0f / s;
    argmax[t] = i;
  }
}

// ---------------------------------------------------------------- a14: commit

struct PolicyDev {
  int kind;       // 0 top-k, 1 threshold
  int k;
  float tau;
  int floor;
  int max_steps;
  int t2t;        // token-to-token editing of committed positions
  float edit_tau;
};

// One CTA per request (C <= 1024 positions). Commits the n most confident masked
// positions (fp32 conf, ties to the lower position): top-k: n = min(k, R);
// threshold: n = max(#{conf > tau}, n_min) with the step-budget floor
// n_min = max(1, ceil(R / (S_max - s))), capped at R. Writes the committed token,
// clears the mask bit, stores R - n and advances the request's step counter. With T2T
// editing on, a position committed before this pass is re-written to the pass's argmax
// when that token differs and conf > edit_tau (the mask and R are left alone). If a
// kernel of the pass gave up a bounded wait (*err != 0), nothing is committed or edited
// and the remaining count is -1.
__global__ void commit_kernel(int32_t* __restrict__ canvas, uint8_t* __restrict__ mask, const float* __restrict__ conf,
                              const int32_t* __restrict__ argmax, int C, const PolicyDev* __restrict__ pol,
                              int32_t* __restrict__ step, int32_t* __restrict__ remaining, float* __restrict__ conf_out,
                              int32_t* __restrict__ argmax_out, const int* __restrict__ err) {
  pdl_begin();
  if (*err) {
    if (threadIdx.x == 0) remaining[blockIdx.x] = -1;
    return;
  }
  extern __shared__ uint8_t smc[];
  float* sc = reinterpret_cast<float*>(smc);
  uint8_t* sm = smc + C * sizeof(float);
  const int b = blockIdx.x, i = threadIdx.x;
  const long o = (long)b * C + i;
  const PolicyDev P = *pol;
  float ci = 0.f;
  int mi = 0;
  if (i < C) {
    ci = conf[o];
    mi = mask[o];
    sc[i] = ci;
    sm[i] = (uint8_t)mi;
    if (conf_out) conf_out[o] = ci;
    if (argmax_out) argmax_out[o] = argmax[o];
  }
  const int R = __syncthreads_count(i < C && mi);
  const int above = __syncthreads_count(i < C && mi && ci > P.tau);
  const int s = step[b];
  int n;
  if (P.kind == 0) {
    n = P.k;
  } else {
    n = above;
    if (P.floor) {
      const int left = P.max_steps - s;
      const int nmin = left <= 0 ? R : max(1, (R + left - 1) / left);
      n = max(n, nmin);
    }
  }
  n = max(0, min(n, R));
  if (i < C && mi) {
    int rank = 0;
    for (int j = 0; j < C; ++j) {
      const float cj = sc[j];
      rank += (sm[j] && (cj > ci || (cj == ci && j < i))) ? 1 : 0;
    }
    if (rank < n) {
      canvas[o] = argmax[o];
      mask[o] = 0;
    }
  }
  if (i < C && !mi && P.t2t) {
    const int a = argmax[o];
    if (a != canvas[o] && ci > P.edit_tau) canvas[o] = a;
  }
  if (i == 0) {
    remaining[b] = R - n;
    step[b] = s + 1;
  }
}

// The step's policy and, for n_steps > 0, the step counters of requests 0..n_steps-1.
// The values arrive as kernel arguments, so the caller keeps no host buffer alive and
// the call needs no synchronisation.
__global__ void stage_step_kernel(PolicyDev pd, int step, int n_steps, PolicyDev* __restrict__ pol,
                                  int32_t* __restrict__ steps) {
  pdl_begin();
  if (threadIdx.x == 0) *pol = pd;
  for (int i = threadIdx.x; i < n_steps; i += blockDim.x) steps[i] = step;
}

// dst[i] = v (add = 0) or dst[i] += v (add = 1) for i < n: prefix lengths and slot ids
// set without a host staging buffer.
__global__ void set_ints_kernel(int32_t* __restrict__ dst, int n, int v, int add) {
  pdl_begin();
  for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = add ? dst[i] + v : v;
}

// After a single GEMM: if a kernel gave up a bounded wait, D is incomplete; fill it
// with NaN so that a caller who cannot wait for an error code still sees it.
__global__ void poison_on_error_kernel(const int* __restrict__ err, float* __restrict__ d, long n) {
  pdl_begin();
  if (!*err) return;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
    d[i] = __int_as_float(0x7fc00000);
}

// Fresh all-[MASK] canvases and zeroed step counters.
__global__ void canvas_init_kernel(int32_t* canvas, uint8_t* mask, int n, int mask_id, int32_t* step, int B) {
  pdl_begin();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    canvas[i] = mask_id;
    mask[i] = 1;
  }
  if (i < B) step[i] = 0;
}

// ---------------------------------------------------------------- FP8 expert weights

// One CTA per 128 x 128 tile (bi, bj) = (blockIdx.y, blockIdx.x) of a bf16 matrix src
// [rows][cols]: the tile's scale exponent e is the least integer with max|w| <= 448 * 2^e
// (0 for an all-zero tile), stored at exps[bi * gridDim.x + bj]; every element becomes the
// E4M3 code of w * 2^-e (round to nearest even), written to dst row
// (i / group) * group_stride + i % group + row_offset (the same row map as
// pack_rows_kernel), dst rows cols bytes long.
__global__ void __launch_bounds__(256) quantize_e4m3_blocks_kernel(const bf16_t* __restrict__ src, int rows, int cols,
                                                                   uint8_t* __restrict__ dst, int8_t* __restrict__ exps,
                                                                   long group, long group_stride, long row_offset) {
  pdl_begin();
  const int r0 = blockIdx.y * 128, c0 = blockIdx.x * 128;
  const int nr = min(128, rows - r0), nc = min(128, cols - c0);
  float amax = 0.f;
  for (int i = threadIdx.x; i < nr * nc; i += blockDim.x) {
    const int r = i / nc, c = i % nc;
    amax = fmaxf(amax, fabsf(bf16_to_f32(src[(long)(r0 + r) * cols + c0 + c])));
  }
  __shared__ float red[8];
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) amax = fmaxf(amax, red[w]);
  int e = 0;
  if (amax > 0.f) {
    e = (int)ceilf(log2f(amax / 448.0f));
    while (amax > ldexpf(448.0f, e)) ++e;
    while (amax <= ldexpf(448.0f, e - 1)) --e;
  }
  if (threadIdx.x == 0) exps[blockIdx.y * gridDim.x + blockIdx.x] = (int8_t)e;
  const float inv = ldexpf(1.0f, -e);
  for (int i = threadIdx.x; i < nr * nc; i += blockDim.x) {
    const long r = r0 + i / nc, c = c0 + i % nc;
    const long drow = (r / group) * group_stride + (r % group) + row_offset;
    dst[drow * cols + c] = f32_to_e4m3(bf16_to_f32(src[r * cols + c]) * inv);
  }
}

// ---------------------------------------------------------------- weight packing

// dst row ((i / group) * group_stride + i % group + row_offset) = bf16(src row i).
__global__ void pack_rows_kernel(bf16_t* __restrict__ dst, const void* __restrict__ src, int src_f32, long n_rows,
                                 int d, long group, long group_stride, long row_offset) {
  const long n = n_rows * d;
  for (long e = (long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long)gridDim.x * blockDim.x) {
    const long i = e / d, c = e % d;
    const long drow = (i / group) * group_stride + (i % group) + row_offset;
    bf16_t v;
    if (src_f32) v = f32_to_bf16(reinterpret_cast<const float*>(src)[e]);
    else v = reinterpret_cast<const bf16_t*>(src)[e];
    dst[drow * d + c] = v;
  }
}

__global__ void to_f32_kernel(float* __restrict__ dst, const void* __restrict__ src, int src_f32, long n) {
  for (long e = (long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long)gridDim.x * blockDim.x) {
    dst[e] = src_f32 ? reinterpret_cast<const float*>(src)[e]
                     : bf16_to_f32(reinterpret_cast<const bf16_t*>(src)[e]);
  }
}

}  // namespace dllm
