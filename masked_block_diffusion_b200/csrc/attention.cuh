// Flash-style attention of canvas (or prompt) queries against the layer's KV cache.
//
// The canvas pass is bidirectional: every query of request b sees all keys
// 0 .. P_b + C - 1, i.e. the cached prefix and the whole canvas, whose K/V the QKV
// epilogue has just written at positions P_b .. P_b + C - 1 (block decoding with a KV
// cache; "Diffusion LLMs: what changes ...", sections 4.1 and 4.2, and the
// bidirectional-attention property of section 2). Prefill is causal (key j visible to
// the query at position i iff j <= i).
//
// One CTA = 64 query rows of one head (4 warps x 16 rows) over one split of the key
// range; keys stream through shared memory in blocks of BK with cp.async double
// buffering; S = Q K^T and O += P V use m16n8k16 bf16 MMAs with fp32 accumulation and
// an online softmax in the exp2 domain. With several splits each CTA writes a partial
// (O / l, log2-sum-exp) and attn_merge_kernel combines them.
#pragma once

#include "common.cuh"

namespace dllm {

// Keys of one split of a request's key range [0, kend): whole 64-key blocks, about
// kend / n_splits of them, so the splits stay balanced whatever the prefix length (the
// last split may be shorter, or empty when kend is small).
DLLM_DEV int split_len(int kend, int n_splits) { return ((kend + n_splits - 1) / n_splits + 63) / 64 * 64; }

struct AttnParams {
  const bf16_t* q;          // [T][H][HD]
  const bf16_t* kc;         // layer cache [slots][Hkv][max_ctx][HD]
  const bf16_t* vc;
  bf16_t* out;              // [T][H*HD] hi part of the output (single split, or after the merge)
  bf16_t* out_lo;           // [T][H*HD] lo part
  float* part_o;            // [splits][T][H][HD]
  float* part_lse;          // [splits][T][H]
  const int* pos0;          // per request: absolute position of query 0
  const int* slot;          // per request: KV slot
  int tok_per_req;          // queries per request
  int T;                    // total query rows
  int H, Hkv, max_ctx;
  int causal;
  int n_splits;
  float scale_log2;         // log2(e) / sqrt(HD)
};

template <int HD, int BK>
struct AttnSmem {
  static constexpr int kStride = HD + 8;     // padded row (bf16) -> conflict-free ldmatrix
  static constexpr int kQ = 64 * kStride * 2;
  static constexpr int kKV = BK * kStride * 2;
  static constexpr int kTotal = kQ + 4 * kKV;
};

// 3 CTAs (12 warps) per SM: Q stays in shared memory and is re-read by ldmatrix per key
// block, which keeps the O accumulators, S tile and temporaries within 170 registers.
template <int HD, int BK>
__global__ void __launch_bounds__(128, 3) attn_kernel(AttnParams p) {
  pdl_begin();
  static_assert(HD % 16 == 0 && BK % 16 == 0, "shape");
  using S = AttnSmem<HD, BK>;
  constexpr int NT = BK / 8;      // S n-tiles per warp
  constexpr int KS = HD / 16;     // k steps of Q K^T
  constexpr int ON = HD / 8;      // O n-tiles
  constexpr int CH = HD / 8;      // 16-byte chunks per row

  extern __shared__ __align__(16) uint8_t sm[];
  bf16_t* sQ = reinterpret_cast<bf16_t*>(sm);
  bf16_t* sK = reinterpret_cast<bf16_t*>(sm + S::kQ);
  bf16_t* sV = reinterpret_cast<bf16_t*>(sm + S::kQ + 2 * S::kKV);

  const int qb = blockIdx.x, h = blockIdx.y;
  const int b = blockIdx.z / p.n_splits, sp = blockIdx.z % p.n_splits;
  const int nq = p.tok_per_req;
  const int q_start = qb * 64;
  if (q_start >= nq) return;
  const int kvh = (h * p.Hkv) / p.H;
  const int P0 = p.pos0[b];
  const int kend = p.causal ? P0 + min(q_start + 64, nq) : P0 + nq;
  const int sk = split_len(kend, p.n_splits);
  const int ks = sp * sk;
  const int ke = min(kend, ks + sk);
  if (ks >= ke) return;
  const int nblk = (ke - ks + BK - 1) / BK;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long tok0 = (long)b * nq;
  const bf16_t* kbase = p.kc + ((long)p.slot[b] * p.Hkv + kvh) * p.max_ctx * HD;
  const bf16_t* vbase = p.vc + ((long)p.slot[b] * p.Hkv + kvh) * p.max_ctx * HD;

  // Q tile: 64 rows (zero rows past the request's queries)
  for (int c = tid; c < 64 * CH; c += 128) {
    const int r = c / CH, ch = c % CH;
    const int qi = q_start + r;
    const bool v = qi < nq;
    const bf16_t* src = p.q + ((tok0 + (v ? qi : 0)) * p.H + h) * HD + ch * 8;
    cp_async16(smem_u32(sQ + r * S::kStride + ch * 8), src, v ? 16 : 0);
  }
  auto load_kv = [&](int blk, int buf) {
    const int k0 = ks + blk * BK;
    for (int c = tid; c < BK * CH; c += 128) {
      const int r = c / CH, ch = c % CH;
      const int key = k0 + r;
      const bool v = key < ke;
      const long off = (long)(v ? key : 0) * HD + ch * 8;
      cp_async16(smem_u32(sK + (buf * BK + r) * S::kStride + ch * 8), kbase + off, v ? 16 : 0);
      cp_async16(smem_u32(sV + (buf * BK + r) * S::kStride + ch * 8), vbase + off, v ? 16 : 0);
    }
  };
  load_kv(0, 0);
  cp_async_commit();

  const int g = lane >> 2, cq = lane & 3;
  const int row0 = warp * 16;
  const int qpos_a = P0 + q_start + row0 + g;   // absolute positions of this thread's rows
  const int qpos_b = qpos_a + 8;

  float o[ON][4];
#pragma unroll
  for (int i = 0; i < ON; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  for (int blk = 0; blk < nblk; ++blk) {
    const int buf = blk & 1;
    if (blk + 1 < nblk) {
      load_kv(blk + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const bf16_t* kb = sK + buf * BK * S::kStride;
    const bf16_t* vb = sV + buf * BK * S::kStride;

    float s[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      uint32_t qf[4];
      {
        const int r = row0 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int c = kk * 16 + 8 * (lane >> 4);
        ldmatrix_x4(qf, smem_u32(sQ + r * S::kStride + c));
      }
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        uint32_t kr[4];
        const int key = np * 16 + (lane & 7) + 8 * (lane >> 4);
        const int c = kk * 16 + 8 * ((lane >> 3) & 1);
        ldmatrix_x4(kr, smem_u32(kb + key * S::kStride + c));
        mma_bf16_16816(s[2 * np], qf, kr[0], kr[1]);
        mma_bf16_16816(s[2 * np + 1], qf, kr[2], kr[3]);
      }
    }
    // scale, mask, block row maxima
    const int k0 = ks + blk * BK;
    float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = k0 + nt * 8 + 2 * cq + (e & 1);
        const int qp = (e < 2) ? qpos_a : qpos_b;
        const bool vis = key < ke && (!p.causal || key <= qp);
        const float v = vis ? s[nt][e] * p.scale_log2 : -INFINITY;
        s[nt][e] = v;
        if (e < 2) mx_a = fmaxf(mx_a, v); else mx_b = fmaxf(mx_b, v);
      }
    }
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
    const float base_a = (mn_a == -INFINITY) ? 0.f : mn_a;
    const float base_b = (mn_b == -INFINITY) ? 0.f : mn_b;
    const float corr_a = exp2f(m_a - base_a), corr_b = exp2f(m_b - base_b);
    m_a = mn_a;
    m_b = mn_b;
    float rs_a = 0.f, rs_b = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      s[nt][0] = exp2f(s[nt][0] - base_a);
      s[nt][1] = exp2f(s[nt][1] - base_a);
      s[nt][2] = exp2f(s[nt][2] - base_b);
      s[nt][3] = exp2f(s[nt][3] - base_b);
      rs_a += s[nt][0] + s[nt][1];
      rs_b += s[nt][2] + s[nt][3];
    }
    l_a = l_a * corr_a + rs_a;
    l_b = l_b * corr_b + rs_b;
#pragma unroll
    for (int i = 0; i < ON; ++i) {
      o[i][0] *= corr_a;
      o[i][1] *= corr_a;
      o[i][2] *= corr_b;
      o[i][3] *= corr_b;
    }
    // O += P V. P is split into P_hi = bf16(P) and P_lo = bf16(P - P_hi) and both are
    // multiplied: near-uniform attention over thousands of keys makes O small, and a
    // single bf16 rounding of P would leave a 2^-9 relative error on it.
#pragma unroll
    for (int kk = 0; kk < BK / 16; ++kk) {
      uint32_t a[4], al[4];
      split_bf16x2(s[2 * kk][0], s[2 * kk][1], a[0], al[0]);
      split_bf16x2(s[2 * kk][2], s[2 * kk][3], a[1], al[1]);
      split_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1], a[2], al[2]);
      split_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3], a[3], al[3]);
#pragma unroll
      for (int np = 0; np < ON / 2; ++np) {
        uint32_t vr[4];
        const int key = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int c = np * 16 + 8 * (lane >> 4);
        ldmatrix_x4_trans(vr, smem_u32(vb + key * S::kStride + c));
        mma_bf16_16816(o[2 * np], a, vr[0], vr[1]);
        mma_bf16_16816(o[2 * np + 1], a, vr[2], vr[3]);
        mma_bf16_16816(o[2 * np], al, vr[0], vr[1]);
        mma_bf16_16816(o[2 * np + 1], al, vr[2], vr[3]);
      }
    }
    __syncthreads();
  }

  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  const float inv_a = l_a > 0.f ? 1.f / l_a : 0.f;
  const float inv_b = l_b > 0.f ? 1.f / l_b : 0.f;
  const int qa = q_start + row0 + g, qbb = qa + 8;
  const bool va = qa < nq, vb2 = qbb < nq;
  const long ta = tok0 + qa, tb = tok0 + qbb;
  if (p.n_splits == 1) {
#pragma unroll
    for (int nt = 0; nt < ON; ++nt) {
      const int c = nt * 8 + 2 * cq;
      uint32_t hi, lo;
      if (va) {
        split_bf16x2(o[nt][0] * inv_a, o[nt][1] * inv_a, hi, lo);
        *reinterpret_cast<uint32_t*>(p.out + (ta * p.H + h) * HD + c) = hi;
        *reinterpret_cast<uint32_t*>(p.out_lo + (ta * p.H + h) * HD + c) = lo;
      }
      if (vb2) {
        split_bf16x2(o[nt][2] * inv_b, o[nt][3] * inv_b, hi, lo);
        *reinterpret_cast<uint32_t*>(p.out + (tb * p.H + h) * HD + c) = hi;
        *reinterpret_cast<uint32_t*>(p.out_lo + (tb * p.H + h) * HD + c) = lo;
      }
    }
  } else {
    float* po = p.part_o + (long)sp * p.T * p.H * HD;
#pragma unroll
    for (int nt = 0; nt < ON; ++nt) {
      const int c = nt * 8 + 2 * cq;
      if (va) *reinterpret_cast<float2*>(po + (ta * p.H + h) * HD + c) = make_float2(o[nt][0] * inv_a, o[nt][1] * inv_a);
      if (vb2) *reinterpret_cast<float2*>(po + (tb * p.H + h) * HD + c) = make_float2(o[nt][2] * inv_b, o[nt][3] * inv_b);
    }
    if (cq == 0) {
      float* pl = p.part_lse + (long)sp * p.T * p.H;
      if (va) pl[ta * p.H + h] = m_a + __log2f(l_a);
      if (vb2) pl[tb * p.H + h] = m_b + __log2f(l_b);
    }
  }
}

// Combines the key splits of a non-causal pass: weights exp2(lse_s - max) per split.
// One warp per (query row, head).
template <int HD>
__global__ void attn_merge_kernel(AttnParams p) {
  pdl_begin();
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= p.T * p.H) return;
  const int t = w / p.H, h = w % p.H;
  const int b = t / p.tok_per_req;
  const int kend = p.pos0[b] + p.tok_per_req;
  const int sk = split_len(kend, p.n_splits);
  const int ns = min(p.n_splits, (kend + sk - 1) / sk);
  float mx = -INFINITY;
  for (int s = 0; s < ns; ++s) mx = fmaxf(mx, p.part_lse[((long)s * p.T + t) * p.H + h]);
  float wsum = 0.f;
  float acc[(HD + 31) / 32];
#pragma unroll
  for (int i = 0; i < (HD + 31) / 32; ++i) acc[i] = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float ws = exp2f(p.part_lse[((long)s * p.T + t) * p.H + h] - mx);
    wsum += ws;
    const float* po = p.part_o + (((long)s * p.T + t) * p.H + h) * HD;
#pragma unroll
    for (int i = 0; i < (HD + 31) / 32; ++i) {
      const int c = lane + 32 * i;
      if (c < HD) acc[i] += ws * po[c];
    }
  }
  const float inv = 1.f / wsum;
#pragma unroll
  for (int i = 0; i < (HD + 31) / 32; ++i) {
    const int c = lane + 32 * i;
    if (c < HD) {
      const float v = acc[i] * inv;
      const bf16_t hi = f32_to_bf16(v);
      p.out[((long)t * p.H + h) * HD + c] = hi;
      p.out_lo[((long)t * p.H + h) * HD + c] = f32_to_bf16(v - bf16_to_f32(hi));
    }
  }
}

}  // namespace dllm
