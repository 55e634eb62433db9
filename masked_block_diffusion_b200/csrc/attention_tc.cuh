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
//
// The split's key blocks are dealt to two independent online-softmax streams: stream 0
// takes the even blocks, stream 1 the odd ones, each with its own running maximum and
// sum, its own O accumulator and its own S buffer in TMEM. While one stream's softmax
// warps turn its scores into probabilities, the tensor pipe runs the other stream's
// S = Q K^T and O += P V, so neither the MMAs nor the softmax wait on each other's whole
// chain. At the end the two streams are merged in log-sum-exp fashion.
//
// Roles (320 threads):
//   warp 0 lane 0  TMA: the Q tile once, then K and V blocks of BK keys, in block order,
//                  into two three-stage rings (a K stage is refilled once the S that read
//                  it completes, a V stage once its P V does);
//   warp 1         TMEM allocation; lane 0 issues the MMAs: S(j) into stream j&1's S
//                  buffer, O_(j&1) += P_hi V + P_lo V once the softmax has written P(j)
//                  over S(j), and S(j+2) into the same buffer once that P V completed;
//   warps 2..5     stream 0's softmax, warps 6..9 stream 1's: one query row per thread
//                  (TMEM lane r), all BK keys of the row per block: read S, scale and
//                  mask, running maximum, P = exp2(s - m_ref) as a bf16 (hi, lo) pair
//                  written back into the S columns with tcgen05.st (the P V MMA reads its
//                  A operand from TMEM), running sum. O is rescaled only when the maximum
//                  grows by more than 2^8 (P stays below 256, exact enough, and rescales
//                  are rare). At the end both streams read O_0 and O_1, merge them and
//                  write the output (or a split partial), each on half of the columns.
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

// Maximum and sum of N register values as a balanced tree (depth log2 N instead of a
// chain of N dependent operations on the softmax's critical path). tree_sum overwrites v.
template <int N>
DLLM_DEV float tree_max(const float (&v)[N]) {
  float a[N / 2];
#pragma unroll
  for (int i = 0; i < N / 2; ++i) a[i] = fmaxf(v[2 * i], v[2 * i + 1]);
#pragma unroll
  for (int w = N / 4; w >= 1; w /= 2)
#pragma unroll
    for (int i = 0; i < w; ++i) a[i] = fmaxf(a[2 * i], a[2 * i + 1]);
  return a[0];
}

template <int N>
DLLM_DEV float tree_sum(float (&v)[N]) {
#pragma unroll
  for (int w = N / 2; w >= 1; w /= 2)
#pragma unroll
    for (int i = 0; i < w; ++i) v[i] = v[2 * i] + v[2 * i + 1];
  return v[0];
}

// True on every softmax thread (both streams, 256 threads, named barrier 1) iff true on
// each of them.
DLLM_DEV bool softmax_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)ok)
      : "memory");
  return r != 0;
}

// TMEM columns: stream s's S buffer at 64 s (P(j) is written over S(j): hi pairs of the
// 64 keys in its first 32 columns, lo pairs in the next 32), O of stream s at 128 + HD s.
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
  static constexpr int kOffRed = kOffBar + 256;          // per stream: (max, sum) of each row, for the merge
  static constexpr int kTotal = kOffRed + 512 * 4 + 1024;
  static constexpr int kSCol = 0;                        // + 64 * stream
  static constexpr int kOCol = 2 * BK;                   // + HD * stream
  static constexpr int kOHalf = ((HD / 2 + 15) / 16) * 16;   // O columns the first stream writes out
  static constexpr int kTmemCols = 512;
  static_assert(kOCol + 2 * HD <= kTmemCols, "TMEM");
  static_assert(kTotal <= 232448, "shared memory");
};

// Warps 2..9: stream st = (warp - 2) / 4; thread (warp w, lane) owns query row
// r = 32 (w % 4) + lane (TMEM lane r) of its stream, all BK keys of each of the stream's
// blocks j = st, st + 2, ...
template <int HD>
DLLM_DEV void softmax_stream(const AttnTcParams& p, uint32_t tmem_base, uint64_t* s_full, uint64_t* p_full,
                             uint64_t* o_final, float* red, volatile int* abort_flag, int warp, int lane, int q0,
                             int b, int sp, int ks, int ke, int nblk) {
  using G = AttnTcCfg<HD>;
  constexpr int BK = G::BK;
  const int q = warp & 3;
  const int st = (warp - 2) >> 2;
  const int r = q * 32 + lane;
  const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
  const uint32_t s_col = lane_base + G::kSCol + st * BK;
  const uint32_t o_own = lane_base + G::kOCol + st * HD;
  // keys this row may see end at row_ke: the tile's end, or (causal) the row's own query
  // position + 1; rows past the last query take the last query's limit (output dropped)
  int row_ke = ke;
  if (p.causal) row_ke = min(ke, p.pos0[b] + min(q0 + r / p.group, p.tok_per_req - 1) + 1);
  float m_ref = -INFINITY, l = 0.f;
  bool ok = true;
  const int nb = (nblk - st + 1) / 2;
  for (int i = 0; i < nb; ++i) {
    const int j = 2 * i + st;
    if (!__all_sync(0xffffffffu, mbar_wait(&s_full[st], i & 1, abort_flag))) { ok = false; break; }
    tc_fence_after();
    float s[BK];
    tmem_ld64(s_col, s);
    const int nvis = row_ke - (ks + j * BK);
    if (nvis < BK) {
#pragma unroll
      for (int c = 0; c < BK; ++c)
        if (c >= nvis) s[c] = -INFINITY;
    }
    // the maximum is taken on the raw scores (scaling by a positive constant commutes
    // with it, rounding included)
    const float mx = tree_max<BK>(s) * p.scale_log2;
    if (i == 0) {
      m_ref = mx;
    } else {
      const bool need = mx > m_ref + 8.0f;
      if (__any_sync(0xffffffffu, need)) {
        // this stream's O is stable here: S(j) was issued only after P V(j - 2) completed
        const float f = need ? exp2f(m_ref - mx) : 1.0f;
#pragma unroll 1
        for (int c = 0; c < HD; c += 16) {
          float v[16];
          tmem_ld16(o_own + c, v);
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] *= f;
          tmem_st16(o_own + c, v);
        }
        if (need) {
          l *= f;
          m_ref = mx;
        }
      }
    }
    // a causal row whose keys so far are all masked has m_ref = -inf: every p is 0
    const float mb = m_ref == -INFINITY ? 0.f : m_ref;
    uint32_t hi[BK / 2], lo[BK / 2];
#pragma unroll
    for (int c = 0; c < BK; c += 2) {
      s[c] = ex2_approx(fmaf(s[c], p.scale_log2, -mb));
      s[c + 1] = ex2_approx(fmaf(s[c + 1], p.scale_log2, -mb));
      split_bf16x2(s[c], s[c + 1], hi[c / 2], lo[c / 2]);
    }
    l += tree_sum<BK>(s);
    // P(j) over S(j): hi pairs of the 64 keys in the buffer's columns 0..31, lo in 32..63
    tmem_st32_nowait(s_col, hi);
    tmem_st32_nowait(s_col + BK / 2, lo);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&p_full[st]);
  }
  if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_final, 0, abort_flag));
  if (!softmax_all(ok)) {
    if (!ok) atomicExch(p.err, kDevTimeoutEpilogue);
    *abort_flag = 1;
    return;
  }
  // merge the two streams per row: each hands its (max, sum) to the other's thread of the
  // same row, then both scale their O by 2^(m_s - m) and each writes half of the columns
  red[st * 256 + r] = m_ref;
  red[st * 256 + 128 + r] = l;
  named_bar_sync(1, 256);
  const float mo = red[(st ^ 1) * 256 + r], lo_other = red[(st ^ 1) * 256 + 128 + r];
  const float m0 = st == 0 ? m_ref : mo, m1 = st == 0 ? mo : m_ref;
  const float l0 = st == 0 ? l : lo_other, l1 = st == 0 ? lo_other : l;
  const float m = fmaxf(m0, m1);
  // a stream that saw no key of this row (or had no block) has m = -inf and adds nothing;
  // its O columns may never have been written, so they are not read into the sum
  const float f0 = m0 == -INFINITY ? 0.f : exp2f(m0 - m);
  const float f1 = m1 == -INFINITY ? 0.f : exp2f(m1 - m);
  const float lt = l0 * f0 + l1 * f1;
  tc_fence_after();
  const int i = r / p.group;
  const int h = blockIdx.y * p.group + r % p.group;
  const bool valid = q0 + i < p.tok_per_req;
  const long t = (long)b * p.tok_per_req + q0 + i;
  const float inv = 1.0f / lt;
  const int c_lo = st == 0 ? 0 : G::kOHalf, c_hi = st == 0 ? G::kOHalf : HD;
  const uint32_t o0 = lane_base + G::kOCol, o1 = o0 + HD;
#pragma unroll 1
  for (int c = c_lo; c < c_hi; c += 16) {
    float v[16], w[16];
    tmem_ld16(o0 + c, v);
    tmem_ld16(o1 + c, w);
    if (!valid) continue;
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = ((f0 != 0.f ? v[e] * f0 : 0.f) + (f1 != 0.f ? w[e] * f1 : 0.f)) * inv;
    if (p.n_splits == 1) {
      uint32_t hw[8], lw[8];
#pragma unroll
      for (int e = 0; e < 16; e += 2) split_bf16x2(v[e], v[e + 1], hw[e / 2], lw[e / 2]);
      bf16_t* oh = p.out + (t * p.H + h) * HD + c;
      bf16_t* ol = p.out_lo + (t * p.H + h) * HD + c;
      reinterpret_cast<uint4*>(oh)[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      reinterpret_cast<uint4*>(oh)[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
      reinterpret_cast<uint4*>(ol)[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      reinterpret_cast<uint4*>(ol)[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
    } else {
      float4* po = reinterpret_cast<float4*>(p.part_o + (((long)sp * p.T + t) * p.H + h) * HD + c);
#pragma unroll
      for (int e = 0; e < 4; ++e) po[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    }
  }
  if (valid && st == 0 && p.n_splits > 1) p.part_lse[((long)sp * p.T + t) * p.H + h] = m + __log2f(lt);
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
  uint64_t* s_full = v_empty + ST;     // [2]: stream s's S(j) is in its buffer
  uint64_t* p_full = s_full + 2;       // [2]: stream s's P(j) is written over it
  uint64_t* pv_done = p_full + 2;      // [2]: stream s's P V(j) completed (its buffer is free)
  uint64_t* o_final = pv_done + 2;
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);   // one arrival per softmax warp of the stream
      mbar_init(&pv_done[i], 1);
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
    // S(jj) = Q K(jj)^T into stream jj&1's buffer
    auto issue_s = [&](int jj) -> bool {
      const int kst = jj % ST, sb = jj & 1;
      if (!mbar_wait(&k_full[kst], (jj / ST) & 1, abort_flag)) return false;
      tc_fence_after();
      const uint32_t d_s = tmem_base + G::kSCol + sb * BK;
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK + kst * G::kKV);
#pragma unroll
      for (int a = 0; a < AT; ++a)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(d_s, sdesc_k_sw128(q_base + a * 128 * 128 + kk * 32),
                    sdesc_k_sw128(k_base + a * G::kKatom + kk * 32), kIdQK, (a | kk) != 0);
      umma_commit(&s_full[sb]);
      umma_commit(&k_empty[kst]);
      return true;
    };
    // O_(jj&1) += P_hi(jj) V(jj) + P_lo(jj) V(jj); the stream's first block overwrites O
    auto issue_pv = [&](int jj) -> bool {
      const int vst = jj % ST, sb = jj & 1, i = jj >> 1;
      if (!mbar_wait(&v_full[vst], (jj / ST) & 1, abort_flag)) return false;
      if (!mbar_wait(&p_full[sb], i & 1, abort_flag)) return false;
      tc_fence_after();
      const uint32_t p_hi = tmem_base + G::kSCol + sb * BK;
      const uint32_t p_lo = p_hi + BK / 2;
      const uint32_t d_o = tmem_base + G::kOCol + sb * HD;
      const uint32_t v0 = smem_u32(sV + vst * G::kKV);
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        const uint64_t bdesc = sdesc_mn_sw128(v0 + kk * 16 * 128, G::kKatom);
        umma_bf16_ts(d_o, p_hi + kk * 8, bdesc, kIdPV, (i | kk) != 0);
        umma_bf16_ts(d_o, p_lo + kk * 8, bdesc, kIdPV, 1);
      }
      umma_commit(&v_empty[vst]);
      umma_commit(&pv_done[sb]);
      return true;
    };
    if (ok && nblk > 0) ok = issue_s(0);
    if (ok && nblk > 1) ok = issue_s(1);
    for (int j = 0; j < nblk && ok; ++j) {
      if (!issue_pv(j)) { ok = false; break; }
      if (j + 2 < nblk) {
        // S(j+2) goes into the columns P V(j) reads: wait until that MMA has completed
        if (!mbar_wait(&pv_done[j & 1], (j >> 1) & 1, abort_flag)) { ok = false; break; }
        if (!issue_s(j + 2)) { ok = false; break; }
      }
    }
    if (ok) umma_commit(o_final);
    if (!ok) {
      atomicExch(p.err, kDevTimeoutMma);
      *abort_flag = 1;
    }
    umma_commit(drain);
    mbar_drain(drain, 0);
  } else if (warp >= 2) {
    softmax_stream<HD>(p, tmem_base, s_full, p_full, o_final, reinterpret_cast<float*>(smem + G::kOffRed),
                       abort_flag, warp, lane, q0, b, sp, ks, ke, nblk);
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
