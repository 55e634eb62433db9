// Tensor-core (tcgen05 / TMEM) attention for the canvas passes and the prompt prefill.
//
// Every canvas query of request b sees keys 0 .. P_b + C - 1: the cached prefix and the
// canvas, whose K/V the QKV epilogue has written at P_b .. P_b + C - 1 ("Diffusion LLMs:
// what changes ...", section 2 property 1 and section 4.2 "Block decoding"). A prompt
// token (causal prefill) sees the keys up to its own position.
//
// One CTA = one 128-row query tile of one KV head over one split of the key range. The
// tile holds the GQA group's heads for 128 / group queries (row r = query r / group,
// head r % group), so each K/V block is loaded once for all heads that read it.
// Roles (320 threads):
//   warp 0 lane 0  TMA: the Q tile once, then K and V blocks of BK keys into two
//                  three-stage rings (a K stage is refilled once the S = Q K^T that read
//                  it completes, a V stage once its P V does);
//   warp 1         TMEM allocation; lane 0 issues S = Q K^T into one of three TMEM S
//                  buffers two blocks ahead of O += P_hi V + P_lo V, so the scores of the
//                  next blocks are ready while the softmax works on the current one;
//   warps 2..9     two warpgroups, each on one half (32 keys) of a block, one query row
//                  per thread in each: read S from TMEM, scale and mask, running
//                  maximum, P = exp2(s - m_ref) as a bf16 (hi, lo) pair written back into
//                  TMEM with tcgen05.st (the P V MMA reads its A operand from TMEM, so P
//                  needs no shared memory), running sum; O in TMEM is rescaled only when
//                  the maximum grows by more than 2^8 (P stays below 256, exact enough,
//                  and rescales are rare). At the end they read O, divide by the sum and
//                  write the output (or a split partial).
// Every wait is bounded, as in gemm_tc.cuh.
#pragma once

#include "common.cuh"
#include "attention.cuh"

namespace dllm {

struct AttnTcParams {
  bf16_t* out;              // [T][H*HD] hi part (single split)
  bf16_t* out_lo;           // [T][H*HD] lo part
  float* part_o;            // [splits][T][H][HD]
  float* part_lse;          // [splits][T][H] (log2 domain)
  const int* pos0;          // per request: prefix length P_b (queries sit at P_b + i)
  const int* slot;          // per request: KV slot
  int tok_per_req;          // canvas positions C
  int T;                    // total query rows
  int H, Hkv, group, max_ctx;
  int n_splits;
  int causal;               // 1: query i of request b sees keys 0 .. P_b + i (prompt prefill)
  float scale_log2;         // log2(e) / sqrt(HD)
  int* err;
};

// Shared-memory descriptor of an MN-major operand stored with the 128-byte swizzle:
// 64 contiguous elements (128 B) along N per row, rows along K 128 B apart, 8-row groups
// 1024 B apart (SBO), 64-element N chunks `lbo` bytes apart (LBO).
DLLM_DEV uint64_t sdesc_mn_sw128(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: bf16 A (K-major) x bf16 B (MN-major), fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16_f32_bmn(int M, int N) {
  return idesc_bf16_f32(M, N) | (1u << 16);
}

DLLM_DEV void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"((uint64_t)map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// 2^x with the hardware approximation (PTX ex2.approx; relative error about 2^-22,
// far below the 2^-16 kept by the (hi, lo) bf16 pair P is stored as). ex2(-inf) = 0.
DLLM_DEV float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// True on both warps of a lane-quarter pair (the two softmax halves of the same rows)
// iff true on each of their 64 threads (named barrier `id`). The pairs agree on leaving
// the loop together without holding the other pairs back.
DLLM_DEV bool pair_all(bool ok, int id) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 64, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)ok), "r"(id)
      : "memory");
  return r != 0;
}

// TMEM columns: S buffers at 0, 64 and 128; P buffer pb at 192 + 64 pb (hi in the first 32
// columns, lo in the next 32, two bf16 per column); O from column 320.
template <int HD>
struct AttnTcCfg {
  static constexpr int BK = 64;
  static constexpr int ATOMS = (HD + 63) / 64;
  static constexpr int STAGES = 3;
  static constexpr int kQ = ATOMS * 128 * 128;
  static constexpr int kKatom = BK * 128;
  static constexpr int kKV = ATOMS * kKatom;
  static constexpr int kOffK = kQ;
  static constexpr int kOffV = kOffK + STAGES * kKV;
  static constexpr int kOffBar = kOffV + STAGES * kKV;
  static constexpr int kOffRed = kOffBar + 256;          // softmax halves: maxima [2][2][128], sums [2][128]
  static constexpr int kTotal = kOffRed + 768 * 4 + 1024;
  static constexpr int kOSplit = ((HD / 2 + 15) / 16) * 16;   // O columns of the first softmax half
  static constexpr int kSBufs = 3;                       // S buffers: S(j+2) is issued before P V(j)
  static constexpr int kSCols = BK;
  static constexpr int kPCol = kSBufs * BK;
  static constexpr int kOCol = kPCol + 2 * BK;
  static constexpr int kTmemCols = 512;
  static_assert(kPCol + 2 * BK <= kOCol && kOCol + HD <= kTmemCols, "TMEM");
  static_assert(kTotal <= 232448, "shared memory");
};

// Warps 2..9: two warpgroups, the first on keys 0..31 of each block, the second on keys
// 32..63; thread (warp w, lane) owns query row r = 32 (w % 4) + lane (TMEM lane r) in
// both, so each row's exponentials are split over two warps of the same SM sub-partition
// pair. The halves agree on the row maximum through shared memory (red[parity][half][r],
// one 64-thread named barrier per lane quarter), so they take the same rescaling
// decisions; each rescales and finally writes its own column range of O, and the row sum
// is combined once at the end.
template <int HD>
DLLM_DEV void softmax_rows(const AttnTcParams& p, uint32_t tmem_base, uint64_t* s_full, uint64_t* s_empty,
                           uint64_t* p_full, uint64_t* p_empty, uint64_t* o_final, float* red,
                           volatile int* abort_flag, int warp, int lane, int q0, int b, int sp, int ks, int ke,
                           int nblk) {
  using G = AttnTcCfg<HD>;
  constexpr int BK = G::BK, HB = BK / 2;   // keys per half
  static_assert(BK == 64, "two 32-key halves per block");
  const int q = warp & 3;
  const int half = (warp - 2) >> 2;
  const int r = q * 32 + lane;
  const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
  const int o_lo = half == 0 ? 0 : G::kOSplit, o_hi = half == 0 ? G::kOSplit : HD;   // this half's O columns
  const int pair_bar = 3 + q;   // named barrier of the two warps sharing lane quarter q
  // keys this row may see end at row_ke: the tile's end, or (causal) the row's own query
  // position + 1; rows past the last query take the last query's limit (output dropped)
  int row_ke = ke;
  if (p.causal) row_ke = min(ke, p.pos0[b] + min(q0 + r / p.group, p.tok_per_req - 1) + 1);
  float m_ref = -INFINITY, l = 0.f;
  bool ok = true;
  for (int j = 0; j < nblk; ++j) {
    const int sb = j % G::kSBufs;
    if (!pair_all(mbar_wait(&s_full[sb], (j / G::kSBufs) & 1, abort_flag), pair_bar)) { ok = false; break; }
    tc_fence_after();
    float s[HB];
    tmem_ld32(lane_base + sb * G::kSCols + half * HB, s);
    tc_fence_before();
    mbar_arrive(&s_empty[sb]);
    // the maximum is taken on the raw scores (scaling by a positive constant commutes
    // with it, rounding included); keys past the row's end are masked only in the
    // blocks that have some
    const int nvis = row_ke - (ks + j * BK + half * HB);
    float mx_raw = -INFINITY;
    if (nvis >= HB) {
#pragma unroll
      for (int c = 0; c < HB; ++c) mx_raw = fmaxf(mx_raw, s[c]);
    } else {
#pragma unroll
      for (int c = 0; c < HB; ++c) {
        if (c >= nvis) s[c] = -INFINITY;
        mx_raw = fmaxf(mx_raw, s[c]);
      }
    }
    float* slot = red + (j & 1) * 256;
    slot[half * 128 + r] = mx_raw;
    named_bar_sync(pair_bar, 64);
    mx_raw = fmaxf(mx_raw, slot[(half ^ 1) * 128 + r]);
    const float mx = mx_raw * p.scale_log2;
    if (j == 0) {
      m_ref = mx;   // block 0 always holds a visible key of every row
    } else {
      const bool need = mx > m_ref + 8.0f;
      if (__any_sync(0xffffffffu, need)) {
        // O is rescaled once P V(j-1) has landed: its completion is the commit on P buffer
        // (j-1)&1 (with S issued ahead of P V, S(j) being ready no longer implies it)
        const bool got =
            __all_sync(0xffffffffu, mbar_wait(&p_empty[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag));
        if (got) {
          tc_fence_after();
          const float f = need ? exp2f(m_ref - mx) : 1.0f;
#pragma unroll 1
          for (int c = o_lo; c < o_hi; c += 16) {
            float v[16];
            tmem_ld16(lane_base + G::kOCol + c, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] *= f;
            tmem_st16(lane_base + G::kOCol + c, v);
          }
          tc_fence_before();
          if (need) {
            l *= f;
            m_ref = mx;
          }
        } else {
          ok = false;
        }
      }
    }
    uint32_t hi[HB / 2], lo[HB / 2];
    float psum = 0.f;
#pragma unroll
    for (int c = 0; c < HB; c += 2) {
      const float p0 = ex2_approx(fmaf(s[c], p.scale_log2, -m_ref));
      const float p1 = ex2_approx(fmaf(s[c + 1], p.scale_log2, -m_ref));
      psum += p0 + p1;
      split_bf16x2(p0, p1, hi[c / 2], lo[c / 2]);
    }
    l += psum;
    const int pb = j & 1;
    if (!pair_all(ok && mbar_wait(&p_empty[pb], ((j >> 1) & 1) ^ 1, abort_flag), pair_bar)) {
      ok = false;
      break;
    }
    tc_fence_after();
    // P buffer pb: hi pairs of keys 0..63 in columns 0..31, lo pairs in 32..63
    const uint32_t pcol = lane_base + G::kPCol + pb * BK + half * (HB / 2);
    tmem_st16_nowait(pcol, hi);
    tmem_st16_nowait(pcol + BK / 2, lo);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&p_full[pb]);
  }
  if (ok) ok = pair_all(mbar_wait(o_final, 0, abort_flag), pair_bar);
  if (!ok) {
    atomicExch(p.err, kDevTimeoutEpilogue);
    *abort_flag = 1;
    return;
  }
  // row sum of both halves
  red[512 + half * 128 + r] = l;
  named_bar_sync(pair_bar, 64);
  l += red[512 + (half ^ 1) * 128 + r];
  tc_fence_after();
  const int i = r / p.group;
  const int h = blockIdx.y * p.group + r % p.group;
  const bool valid = q0 + i < p.tok_per_req;
  const long t = (long)b * p.tok_per_req + q0 + i;
  const float inv = 1.0f / l;
#pragma unroll 1
  for (int c = o_lo; c < o_hi; c += 16) {
    float v[16];
    tmem_ld16(lane_base + G::kOCol + c, v);
    if (!valid) continue;
    if (p.n_splits == 1) {
      uint32_t hw[8], lw[8];
#pragma unroll
      for (int e = 0; e < 16; e += 2) split_bf16x2(v[e] * inv, v[e + 1] * inv, hw[e / 2], lw[e / 2]);
      bf16_t* oh = p.out + (t * p.H + h) * HD + c;
      bf16_t* ol = p.out_lo + (t * p.H + h) * HD + c;
      reinterpret_cast<uint4*>(oh)[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      reinterpret_cast<uint4*>(oh)[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
      reinterpret_cast<uint4*>(ol)[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      reinterpret_cast<uint4*>(ol)[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
    } else {
      float4* po = reinterpret_cast<float4*>(p.part_o + (((long)sp * p.T + t) * p.H + h) * HD + c);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        po[e] = make_float4(v[4 * e] * inv, v[4 * e + 1] * inv, v[4 * e + 2] * inv, v[4 * e + 3] * inv);
    }
  }
  if (valid && half == 0 && p.n_splits > 1) p.part_lse[((long)sp * p.T + t) * p.H + h] = m_ref + __log2f(l);
}

template <int HD>
__global__ void __launch_bounds__(320, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, AttnTcParams p) {
  using G = AttnTcCfg<HD>;
  constexpr int BK = G::BK, AT = G::ATOMS, ST = G::STAGES;
  constexpr uint32_t kIdQK = idesc_bf16_f32(128, BK);
  constexpr uint32_t kIdPV = idesc_bf16_f32_bmn(128, HD);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + G::kOffK;
  uint8_t* sV = smem + G::kOffV;
  uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + G::kOffBar);
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + ST;
  uint64_t* v_full = k_empty + ST;
  uint64_t* v_empty = v_full + ST;
  uint64_t* s_full = v_empty + ST;
  uint64_t* s_empty = s_full + G::kSBufs;
  uint64_t* p_full = s_empty + G::kSBufs;
  uint64_t* p_empty = p_full + 2;
  uint64_t* o_final = p_empty + 2;
  uint64_t* drain = o_final + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  pdl_wait();   // pos0 and the K / V written by the QKV projection
  // causal: the last query tiles see the most keys, so they are launched first
  const int qt = p.causal ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x, g = blockIdx.y;
  const int b = blockIdx.z / p.n_splits, sp = blockIdx.z % p.n_splits;
  const int C = p.tok_per_req, grp = p.group;
  const int qpt = 128 / grp;
  const int q0 = qt * qpt;
  const int kend = p.pos0[b] + (p.causal ? min(C, q0 + qpt) : C);
  const int sk = split_len(kend, p.n_splits);
  const int ks = sp * sk;
  const int ke = min(kend, ks + sk);
  if (q0 >= C || ks >= ke) return;   // uniform over the CTA, before any barrier or TMEM use
  const int nblk = (ke - ks + BK - 1) / BK;
  const int kv_row0 = (p.slot[b] * p.Hkv + g) * p.max_ctx;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int i = 0; i < G::kSBufs; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 256);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&p_full[i], 256);
      mbar_init(&p_empty[i], 1);
    }
    mbar_init(o_final, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, G::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_trigger();   // after the TMEM allocation
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer: K(j) and V(j) in order, each into its own ring
    const uint64_t pol = policy_evict_last();
    bool ok = true;
    int k_issued = 0, v_issued = 0;   // K and V blocks whose loads were issued
    mbar_arrive_expect_tx(q_full, G::kQ);
    for (int a = 0; a < AT; ++a) tma_load_3d(sQ + a * 128 * 128, &tm_q, q_full, a * 64, g * grp, b * C + q0);
    for (int j = 0; j < nblk && ok; ++j) {
      const int st = j % ST;
      const uint32_t ph = ((j / ST) & 1) ^ 1;
      const int row = kv_row0 + ks + j * BK;
      if (!mbar_wait(&k_empty[st], ph, abort_flag)) { ok = false; break; }
      mbar_arrive_expect_tx(&k_full[st], G::kKV);
      for (int a = 0; a < AT; ++a) tma_load_2d(sK + st * G::kKV + a * G::kKatom, &tm_k, &k_full[st], a * 64, row, pol);
      k_issued = j + 1;
      if (!mbar_wait(&v_empty[st], ph, abort_flag)) { ok = false; break; }
      mbar_arrive_expect_tx(&v_full[st], G::kKV);
      for (int a = 0; a < AT; ++a) tma_load_2d(sV + st * G::kKV + a * G::kKatom, &tm_v, &v_full[st], a * 64, row, pol);
      v_issued = j + 1;
    }
    if (!ok) {
      atomicExch(p.err, kDevTimeoutProducer);
      *abort_flag = 1;
      // the loads already issued land before the CTA's shared memory goes away: the
      // Q tile and the last fill of each K and V stage
      mbar_drain(q_full, 0);
      for (int jj = max(0, k_issued - ST); jj < k_issued; ++jj) mbar_drain(&k_full[jj % ST], (jj / ST) & 1);
      for (int jj = max(0, v_issued - ST); jj < v_issued; ++jj) mbar_drain(&v_full[jj % ST], (jj / ST) & 1);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    bool ok = mbar_wait(q_full, 0, abort_flag);
    const uint32_t d_o = tmem_base + G::kOCol;
    auto issue_pv = [&](int jj) -> bool {
      const int pb = jj & 1, st = jj % ST;
      if (!mbar_wait(&v_full[st], (jj / ST) & 1, abort_flag)) return false;
      if (!mbar_wait(&p_full[pb], (jj >> 1) & 1, abort_flag)) return false;
      tc_fence_after();
      const uint32_t p_hi = tmem_base + G::kPCol + pb * BK;
      const uint32_t p_lo = p_hi + BK / 2;
      const uint32_t v0 = smem_u32(sV + st * G::kKV);
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        const uint64_t bdesc = sdesc_mn_sw128(v0 + kk * 16 * 128, G::kKatom);
        umma_bf16_ts(d_o, p_hi + kk * 8, bdesc, kIdPV, (jj | kk) != 0);
        umma_bf16_ts(d_o, p_lo + kk * 8, bdesc, kIdPV, 1);
      }
      umma_commit(&p_empty[pb]);
      umma_commit(&v_empty[st]);
      return true;
    };
    // S = Q K^T for block jj into S buffer jj % kSBufs
    auto issue_s = [&](int jj) -> bool {
      const int st = jj % ST, sb = jj % G::kSBufs;
      if (!mbar_wait(&k_full[st], (jj / ST) & 1, abort_flag)) return false;
      if (!mbar_wait(&s_empty[sb], ((jj / G::kSBufs) & 1) ^ 1, abort_flag)) return false;
      tc_fence_after();
      const uint32_t d_s = tmem_base + sb * G::kSCols;
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK + st * G::kKV);
#pragma unroll
      for (int a = 0; a < AT; ++a)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(d_s, sdesc_k_sw128(q_base + a * 128 * 128 + kk * 32),
                    sdesc_k_sw128(k_base + a * G::kKatom + kk * 32), kIdQK, (a | kk) != 0);
      umma_commit(&s_full[sb]);
      umma_commit(&k_empty[st]);
      return true;
    };
    // S runs kSBufs - 1 blocks ahead of P V, so the tensor pipe always has the next
    // scores queued while the softmax warps work on the current block
    constexpr int kAhead = G::kSBufs - 1;
    for (int j = 0; j < kAhead && j < nblk && ok; ++j) ok = issue_s(j);
    for (int j = 0; j < nblk && ok; ++j) {
      if (j + kAhead < nblk && !issue_s(j + kAhead)) { ok = false; break; }
      if (!issue_pv(j)) { ok = false; break; }
    }
    if (ok) umma_commit(o_final);
    if (!ok) {
      atomicExch(p.err, kDevTimeoutMma);
      *abort_flag = 1;
    }
    umma_commit(drain);
    mbar_drain(drain, 0);
  } else if (warp >= 2) {
    softmax_rows<HD>(p, tmem_base, s_full, s_empty, p_full, p_empty, o_final,
                     reinterpret_cast<float*>(smem + G::kOffRed), abort_flag, warp, lane, q0, b, sp, ks, ke, nblk);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, G::kTmemCols);
  }
}

}  // namespace dllm
