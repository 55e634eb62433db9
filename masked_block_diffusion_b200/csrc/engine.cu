// libdllm: the masked block-diffusion denoiser behind a C ABI (include/dllm.h).
//
// Per canvas pass (What changes, section 2 "Reverse (generation) process"; section 4.2
// "Block decoding"), for T = B * C canvas tokens:
//   embed -> per layer [ RMSNorm -> QKV GEMM (+RoPE, K/V into the cache at P..P+C-1)
//   -> bidirectional attention over [prefix | canvas] -> O GEMM (+residual) -> RMSNorm
//   -> fp32 router + top-k -> permute -> gather -> grouped gate/up GEMM (+SwiGLU)
//   -> grouped down GEMM -> combine (+residual) ] -> final RMSNorm -> LM-head GEMM with
//   fused max / argmax / sum-exp -> merge -> commit.
// The same layer pipeline runs the causal prefill and the append pass. A canvas pass
// is captured once per batch size into a CUDA graph and replayed every step.

#include "dllm.h"

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "attention.cuh"
#include "attention_tc.cuh"
#include "common.cuh"
#include "gemm_tc.cuh"
#include "kernels.cuh"

using namespace dllm;

namespace {

// NVTX range for the duration of a scope: entry points and, when kernels are launched
// eagerly (graph capture, DLLM_NO_GRAPH), each layer. A no-op unless a profiler attaches.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows][cols] matrix, box = 64 columns x box_rows,
// 128-byte swizzle (the layout the UMMA shared-memory descriptors expect).
// 3-D bf16 tensor map over [d2][d1][d0] (d0 contiguous), box = 64 x b1 x b2, 128-byte swizzle.
bool make_tmap3(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b1, uint32_t b2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (d0 * 2) % 16 || b1 == 0 || b1 > 256 || b2 == 0 || b2 > 256)
    return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {64, b1, b2};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (cols * 2) % 16 || box_rows == 0 || box_rows > 256) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D uint8 tensor map over [rows][cols] FP8 codes, box = 64 columns x box_rows, 64-byte
// swizzle (the converter warps read each row's four 16-byte chunks at chunk ^ ((row >> 1) & 3)).
bool make_tmap_u8(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || cols % 16 || box_rows == 0 || box_rows > 256) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Token-operand boxes of the grouped expert GEMMs: a chunk of up to 64 or 128 tokens is
// loaded from boxes of these heights (its count rounded up to 16), so the MMA width
// follows the chunk's token count.
constexpr int kMoeBN[4] = {16, 32, 64, 128};

// Chunk width of the grouped expert GEMMs: 64 tokens while the mean per expert stays at
// or below 64 (a batch-1 canvas: experts are few and uneven, and more, smaller items
// spread better over the SMs), else 128 (prefill, large batches: fewer weight-tile reads).
int moe_chunk(int N, int E) { return (double)N / (double)E <= 64.0 ? 64 : 128; }

struct LayerW {
  float* attn_norm = nullptr;
  float* ffn_norm = nullptr;
  bf16_t* wqkv = nullptr;   // [(H + 2 Hkv) * hd][d]: Q heads, K heads, V heads
  bf16_t* wo = nullptr;     // [d][H * hd]
  bf16_t* wr = nullptr;     // [E][d]
  bf16_t* wgu = nullptr;    // [E][2F][d]: per 128-row block, 64 gate rows then the 64 matching up rows
  bf16_t* wd = nullptr;     // [E][d][F]
  // FP8 experts (expert_format = DLLM_EXPERTS_FP8): the same layouts as E4M3 codes, and the
  // scale exponents of each 128 x 128 tile of the original Wg / Wu ([E][2][F/128][d/128])
  // and Wd ([E][d/128][F/128]), tile counts rounded up
  uint8_t* wgu8 = nullptr;
  uint8_t* wd8 = nullptr;
  int8_t* egu = nullptr;
  int8_t* ed = nullptr;
  CUtensorMap tm_wqkv, tm_wo, tm_wo128, tm_wgu, tm_wd, tm_wr, tm_wgu8, tm_wd8;
  CUtensorMap tm_k, tm_v;   // this layer's K / V cache as [slot][Hkv][max_ctx] rows of hd
};

struct Graph {
  cudaGraphExec_t exec = nullptr;
  long long kernels = 0;
};

}  // namespace

struct dllm_handle {
  dllm_config c{};
  cudaStream_t st = nullptr;
  bool own_stream = false;
  std::string err;
  int E = 1, k = 1;          // experts and top-k as run (dense: 1, 1)
  bool dense = true;
  int qkv_heads = 0;
  int num_sms = 148;
  long long launches = 0;
  std::vector<void*> allocs;

  bf16_t* emb = nullptr;
  bf16_t* head = nullptr;
  float* final_norm = nullptr;
  CUtensorMap tm_head;
  std::vector<LayerW> L;
  float* rope_cos = nullptr;
  float* rope_sin = nullptr;

  bf16_t* kcache = nullptr;
  bf16_t* vcache = nullptr;
  size_t kv_layer = 0;      // elements per layer: max_batch * Hkv * max_ctx * hd

  int T_max = 0, N_max = 0, T_canvas_max = 0;
  float* x = nullptr;
  bf16_t* y = nullptr;
  float* rstd = nullptr;
  bf16_t* q = nullptr;
  bf16_t* ao = nullptr;
  float* apart = nullptr;
  float* alse = nullptr;
  float* rlogits = nullptr;
  float* rpart = nullptr;     // router GEMM split-K partials, summed by the top-k kernel
  float* opart = nullptr;     // O projection split-K partials, summed by the FFN norm
  long rpart_elems = 0, opart_elems = 0;
  int32_t* tk_idx = nullptr;
  float* tk_w = nullptr;
  int32_t* offsets = nullptr;
  int32_t* slot_of = nullptr;
  int32_t* row_token = nullptr;
  bf16_t* xg = nullptr;
  bf16_t* hbuf = nullptr;
  float* obuf = nullptr;
  float* lm_m = nullptr;
  float* lm_s = nullptr;
  int32_t* lm_i = nullptr;
  float* conf = nullptr;
  int32_t* argmax = nullptr;
  // lo halves of the activation operands carried as (hi, lo) bf16 pairs
  bf16_t* y_lo = nullptr;
  bf16_t* y_lo2 = nullptr;   // third term of the attention norm's output (the QKV operand)
  bf16_t* ao_lo = nullptr;
  bf16_t* xg_lo = nullptr;
  bf16_t* hbuf_lo = nullptr;
  CUtensorMap tm_y, tm_xg[4], tm_h[4];
  CUtensorMap tm_y_lo, tm_y_lo2, tm_xg_lo[4], tm_h_lo[4];
  TokMaps tok_xg, tok_h;     // the grouped GEMMs' token-operand maps: boxes of 16..128 rows, hi then lo
  CUtensorMap tm_ao64, tm_ao64_lo;   // attention output as 64-row boxes (swapped O projection)
  CUtensorMap tm_ao128, tm_ao128_lo; // 128-row boxes (the O projection's split-K tiles)
  CUtensorMap tm_q3;        // q buffer [T][H][hd], box = 64 dims x group heads x 128/group queries
  bool attn_tc = false;     // attention on the tensor cores (the GQA group divides a 128-row query tile)
  bool moe_pair = true;     // grouped down GEMM at BN = 64: two weight tiles per work item
  bool router_tc = false;   // router logits on the tensor cores (experts a multiple of 32)
  bool w8 = false;          // FP8 expert weights

  std::vector<int> P;        // prefix length per slot (-1 = no prefill yet)
  std::vector<char> passed;  // per slot: a canvas pass wrote K/V at P..P+C-1 since the last prefill / append
  int32_t* d_P = nullptr;    // [max_batch]
  int32_t* d_slot = nullptr; // [max_batch] = 0..max_batch-1
  int32_t* d_pre_pos = nullptr;   // [1] = 0
  int32_t* d_pre_slot = nullptr;  // [1]
  int32_t* d_tokens = nullptr;    // prompt staging [T_max]
  int32_t* canvas = nullptr;      // [max_batch][C]
  uint8_t* mask = nullptr;
  int32_t* d_step = nullptr;
  int32_t* d_remaining = nullptr;
  PolicyDev* d_policy = nullptr;
  int32_t* h_remaining = nullptr; // pinned [max_batch]
  int* d_err = nullptr;
  int last_B = 0;

  bool debug = false;
  float* dbg_logits = nullptr;   // [L][T_canvas_max][E]
  int32_t* dbg_idx = nullptr;    // [L][T_canvas_max][k]
  float* dbg_x = nullptr;        // [T_canvas_max][d]
  float* dbg_xl = nullptr;       // [L][T_canvas_max][d] residual after each layer
  int32_t* dbg_force = nullptr;  // [L][force_T][k] experts to use instead of the router's
  bool force_routing = false;
  int force_T = 0;               // token count of the passes the forced routing applies to

  std::map<int, Graph> graphs;   // key: B * 2 + mode

  bool timing = false;
  std::vector<cudaEvent_t> tev;  // [kind][layer][start, stop]
  uint32_t tmask = 0;            // kinds timed (bit k = DLLM_TIMING kind k)
  int tstride = 1;          // time layers l % tstride == 0 only
  double t_ms[DLLM_TIMING_KINDS] = {};
  long long t_n[DLLM_TIMING_KINDS] = {};
  double t_bytes[DLLM_TIMING_KINDS] = {};   // algorithmic bytes of the timed launches
  int32_t* routed = nullptr;        // [E] experts with tokens in the current layer
  int32_t* n_routed = nullptr;      // [1]
  int32_t* chunk_prefix = nullptr;  // [E+1] chunk-count prefix over the routed experts
  int32_t* routed_stat = nullptr;   // [L] n_routed per layer of the last timed pass
  int last_T = 0;                   // tokens of the last timed pass
};

namespace {

int fail(dllm_handle* h, int code, const std::string& msg) {
  if (h) h->err = msg;
  return code;
}

int cuda_fail(dllm_handle* h, cudaError_t e, const char* what) {
  return fail(h, DLLM_E_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define CK(call)                                              \
  do {                                                        \
    cudaError_t e_ = (call);                                  \
    if (e_ != cudaSuccess) return cuda_fail(h, e_, #call);    \
  } while (0)

long g_alloc_count = 0;

// Device allocation tracked by the handle. DLLM_FAULT_ALLOC_AT=n makes the n-th
// allocation of the process fail (host-side fault injection for the error paths).
template <class T>
int dalloc(dllm_handle* h, T** p, size_t count) {
  *p = nullptr;
  ++g_alloc_count;
  const char* f = getenv("DLLM_FAULT_ALLOC_AT");
  if (f && atol(f) == g_alloc_count) return fail(h, DLLM_E_OOM, "injected allocation failure");
  size_t bytes = count * sizeof(T);
  if (bytes == 0) bytes = 16;
  void* v = nullptr;
  cudaError_t e = cudaMalloc(&v, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(h, DLLM_E_OOM, std::string("cudaMalloc: ") + cudaGetErrorString(e));
  }
  h->allocs.push_back(v);
  *p = reinterpret_cast<T*>(v);
  return DLLM_OK;
}

#define DA(ptr, n)                           \
  do {                                       \
    int r_ = dalloc(h, &(ptr), (size_t)(n)); \
    if (r_) return r_;                       \
  } while (0)

int ceil_div(long a, long b) { return (int)((a + b - 1) / b); }

// Threads of a one-row-per-block kernel over d floats: one float4 column each (up to
// 1024), so that all of a row's loads are in flight at once.
int row_threads(int d) { return std::min(1024, (d / 4 + 31) / 32 * 32); }

int attn_splits(const dllm_handle* h, int B) {
  if (h->attn_tc) {
    // tensor-core kernel: one CTA per SM, aim at a single full wave
    const int group = h->c.n_heads / h->c.n_kv_heads;
    const int ctas = ceil_div((long)h->c.canvas * group, 128) * h->c.n_kv_heads * B;
    int s = h->num_sms / ctas;
    return s < 1 ? 1 : (s > 16 ? 16 : s);
  }
  const int qblocks = ceil_div(h->c.canvas, 64);
  const int ctas = qblocks * h->c.n_heads * B;
  int s = ceil_div(2 * 148, ctas);
  if (s < 1) s = 1;
  if (s > 16) s = 16;
  return s;
}

// ------------------------------------------------------------------ launch helpers

// Launches kern on the handle's stream; the launch carries programmatic stream
// serialisation, so the kernel may start while its predecessor drains (every
// kernel of the pass waits for its predecessor with griddepcontrol.wait before its first
// global-memory access).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(dllm_handle* h, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = h->st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}


template <int BN, int STAGES, int ACC, int SPLIT, class Sched, class Epi>
cudaError_t launch_gemm(dllm_handle* h, dim3 grid, const CUtensorMap& ta, const CUtensorMap& tb, int kblocks,
                        int a_first, const Sched& s, const Epi& e, const CUtensorMap* ta2 = nullptr,
                        const CUtensorMap* tb2 = nullptr, const TokMaps* tok = nullptr,
                        const CUtensorMap* ta3 = nullptr) {
  static const TokMaps no_tok{};   // the token maps of a dynamic-width schedule, or the third A term
  TokMaps tk = tok ? *tok : no_tok;
  if (ta3) tk.m[0] = *ta3;
  auto kern = gemm_tc_kernel<BN, STAGES, ACC, SPLIT, Sched, Epi>;
  constexpr int smem = GemmSmem<BN, STAGES, SPLIT, Epi, Sched>::kTotal;
  static_assert(smem <= 232448, "shared memory per CTA");
  cudaError_t r = cudaFuncSetAttribute(reinterpret_cast<const void*>(kern),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (r != cudaSuccess) return r;
  if constexpr (Sched::kKSplit > 1) {
    // split-K: clusters of kKSplit consecutive CTAs share one output tile
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(gemm_threads<Sched>());
    cfg.dynamicSmemBytes = smem;
    cfg.stream = h->st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = Sched::kKSplit;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    if (grid.x % Sched::kKSplit || kblocks < Sched::kKSplit) return cudaErrorInvalidValue;
    r = cudaLaunchKernelEx(&cfg, kern, ta, ta2 ? *ta2 : ta, tb, tb2 ? *tb2 : tb, tk, kblocks, a_first, s, e, h->d_err);
    h->launches++;
    if (r != cudaSuccess) return r;
    return cudaGetLastError();
  }
  r = launch_k(h, kern, grid, dim3(gemm_threads<Sched>()), smem, ta, ta2 ? *ta2 : ta, tb, tb2 ? *tb2 : tb, tk,
               kblocks, a_first, s, e, h->d_err);
  h->launches++;
  if (r != cudaSuccess) return r;
  return cudaGetLastError();
}

// The QKV projection reads the attention norm's output as three bf16 terms (all of its
// fp32 bits, three MMAs per k step): Q, K and V are rounded to bf16 right after, and a
// 16-bit operand would move that rounding often enough to shift attention over
// thousands of cached keys measurably (router logits by up to 2e-3 at a 4096-token prefix).
template <int HD>
cudaError_t qkv_gemm_hd(dllm_handle* h, const LayerW& L, bf16_t* kc, bf16_t* vc, int T, const int* pos0,
                        const int* slot, int tok_per_req) {
  const auto& c = h->c;
  EpiQKV<HD> e{h->q, kc, vc, h->rope_cos, h->rope_sin, pos0, slot, tok_per_req, c.n_heads, c.n_kv_heads, c.max_ctx};
  const int mt = ceil_div(T, 128);
  constexpr int STAGES = HD > 128 ? 3 : 4;
  if (mt * h->qkv_heads * 2 <= 2 * h->num_sms) {
    // few tiles (one canvas): split K over CTA pairs so that about twice as many SMs stream
    DenseSplitKSched<2> s{T, mt, HD};
    return launch_gemm<HD, STAGES, 1, kSplitA3>(h, dim3(mt * h->qkv_heads * 2), h->tm_y, L.tm_wqkv, c.d_model / 64, 0,
                                                s, e, &h->tm_y_lo, nullptr, nullptr, &h->tm_y_lo2);
  }
  DenseSched s{T, mt, HD};
  return launch_gemm<HD, STAGES, 1, kSplitA3>(h, dim3(mt * h->qkv_heads), h->tm_y, L.tm_wqkv, c.d_model / 64, 0, s, e,
                                              &h->tm_y_lo, nullptr, nullptr, &h->tm_y_lo2);
}

cudaError_t qkv_gemm(dllm_handle* h, const LayerW& L, bf16_t* kc, bf16_t* vc, int T, const int* pos0,
                     const int* slot, int tok_per_req) {
  if (h->c.head_dim == 176) return qkv_gemm_hd<176>(h, L, kc, vc, T, pos0, slot, tok_per_req);
  return qkv_gemm_hd<64>(h, L, kc, vc, T, pos0, slot, tok_per_req);
}

template <int HD, int BK>
cudaError_t attention_hd(dllm_handle* h, bf16_t* kc, bf16_t* vc, int T, int nreq, int tok_per_req, const int* pos0,
                         const int* slot, int causal, int splits) {
  const auto& c = h->c;
  AttnParams p;
  p.q = h->q;
  p.kc = kc;
  p.vc = vc;
  p.out = h->ao;
  p.out_lo = h->ao_lo;
  p.part_o = h->apart;
  p.part_lse = h->alse;
  p.pos0 = pos0;
  p.slot = slot;
  p.tok_per_req = tok_per_req;
  p.T = T;
  p.H = c.n_heads;
  p.Hkv = c.n_kv_heads;
  p.max_ctx = c.max_ctx;
  p.causal = causal;
  p.n_splits = splits;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  constexpr int smem = AttnSmem<HD, BK>::kTotal;
  cudaError_t r = cudaFuncSetAttribute(reinterpret_cast<const void*>(attn_kernel<HD, BK>),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (r != cudaSuccess) return r;
  dim3 grid(ceil_div(tok_per_req, 64), c.n_heads, nreq * splits);
  r = launch_k(h, attn_kernel<HD, BK>, grid, dim3(128), smem, p);
  h->launches++;
  if (r != cudaSuccess) return r;
  if (splits > 1) {
    r = launch_k(h, attn_merge_kernel<HD>, dim3(ceil_div((long)T * c.n_heads * 32, 256)), dim3(256), 0, p);
    h->launches++;
    if (r != cudaSuccess) return r;
  }
  return cudaGetLastError();
}

template <int HD>
cudaError_t attention_tc_hd(dllm_handle* h, const LayerW& L, int T, int nreq, int tok_per_req, const int* pos0,
                            const int* slot, int causal, int splits) {
  const auto& c = h->c;
  AttnTcParams p;
  p.out = h->ao;
  p.out_lo = h->ao_lo;
  p.part_o = h->apart;
  p.part_lse = h->alse;
  p.pos0 = pos0;
  p.slot = slot;
  p.tok_per_req = tok_per_req;
  p.causal = causal;
  p.T = T;
  p.H = c.n_heads;
  p.Hkv = c.n_kv_heads;
  p.group = c.n_heads / c.n_kv_heads;
  p.max_ctx = c.max_ctx;
  p.n_splits = splits;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  p.err = h->d_err;
  dim3 grid(ceil_div((long)tok_per_req * p.group, 128), c.n_kv_heads, nreq * splits);
  constexpr int smem = AttnTcCfg<HD>::kTotal;
  cudaError_t r = cudaFuncSetAttribute(reinterpret_cast<const void*>(attn_tc_kernel<HD>),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (r != cudaSuccess) return r;
  r = launch_k(h, attn_tc_kernel<HD>, grid, dim3(320), smem, h->tm_q3, L.tm_k, L.tm_v, p);
  h->launches++;
  if (r != cudaSuccess) return r;
  if (splits > 1) {
    AttnParams m;
    m.out = h->ao;
    m.out_lo = h->ao_lo;
    m.part_o = h->apart;
    m.part_lse = h->alse;
    m.pos0 = pos0;
    m.tok_per_req = tok_per_req;
    m.T = T;
    m.H = c.n_heads;
    m.n_splits = splits;
    r = launch_k(h, attn_merge_kernel<HD>, dim3(ceil_div((long)T * c.n_heads * 32, 256)), dim3(256), 0, m);
    h->launches++;
    if (r != cudaSuccess) return r;
  }
  return cudaGetLastError();
}

cudaError_t attention(dllm_handle* h, bf16_t* kc, bf16_t* vc, int T, int nreq, int tok_per_req, const int* pos0,
                      const int* slot, int causal, int splits, const LayerW* L = nullptr) {
  // tensor cores: the bidirectional canvas pass, and (one key range per query tile) the
  // causal prompt prefill
  if (h->attn_tc && L && (!causal || splits == 1)) {
    if (h->c.head_dim == 176)
      return attention_tc_hd<176>(h, *L, T, nreq, tok_per_req, pos0, slot, causal, splits);
    return attention_tc_hd<64>(h, *L, T, nreq, tok_per_req, pos0, slot, causal, splits);
  }
  if (h->c.head_dim == 176)
    return attention_hd<176, 32>(h, kc, vc, T, nreq, tok_per_req, pos0, slot, causal, splits);
  return attention_hd<64, 64>(h, kc, vc, T, nreq, tok_per_req, pos0, slot, causal, splits);
}

// Event of (kind, layer, start|stop); recorded only when the pass is timed.
cudaError_t tmark(dllm_handle* h, uint32_t tmask, int kind, int layer, int which) {
  if (!(tmask & (1u << kind))) return cudaSuccess;
  if (layer % h->tstride) return cudaSuccess;
  cudaEvent_t ev = h->tev[((size_t)kind * h->c.n_layers + layer) * 2 + which];
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t r = cudaStreamIsCapturing(h->st, &cs);
  if (r != cudaSuccess) return r;
  // under stream capture the record must be "external" to become an event node of the
  // graph (a plain record would only express a dependency); outside capture it is plain
  if (cs == cudaStreamCaptureStatusActive) return cudaEventRecordWithFlags(ev, h->st, cudaEventRecordExternal);
  return cudaEventRecord(ev, h->st);
}

// Router logits on the tensor cores: logits[T][E] = y W_r^T with the normalised
// activations as their (hi, lo) bf16 pair, so each product keeps about 16 mantissa bits
// of y and the sum is fp32. Experts form 32-column tiles; with few tiles (one canvas:
// 2 x 4) the K loop is split over up to 8 independent CTAs (slices x tiles <= 2 x the
// SM count) whose partial logits the top-k kernel adds (*nparts > 0); otherwise the GEMM
// writes the logits itself.
cudaError_t router_gemm(dllm_handle* h, const LayerW& L, int T, int* nparts) {
  const int mt = ceil_div(T, 128);
  const int tiles = mt * (h->E / 32);
  const int kb = h->c.d_model / 64;
  const int ks = std::min({8, kb / 2, 2 * h->num_sms / tiles});
  *nparts = 0;
  if (ks >= 2 && (long)ks * T * h->E <= h->rpart_elems) {
    EpiStoreF32<32> e{h->rpart, h->E, h->E, (long)T * h->E};
    DensePartKSched s{T, mt, 32, ks};
    *nparts = ks;
    return launch_gemm<32, 6, 1, kSplitA>(h, dim3(tiles * ks), h->tm_y, L.tm_wr, kb, 0, s, e, &h->tm_y_lo);
  }
  EpiStoreF32<32> e{h->rlogits, h->E, h->E};
  DenseSched s{T, mt, 32};
  return launch_gemm<32, 6, 1, kSplitA>(h, dim3(tiles), h->tm_y, L.tm_wr, kb, 0, s, e, &h->tm_y_lo);
}

// Attention output projection with the residual add, x += ao * Wo^T, operands swapped:
// weight rows (output features) are M and token chunks N, with the token operand's
// (hi, lo) halves stacked into one MMA of width 2 BN, so each weight tile is read from
// shared memory once per k step (measured faster than tokens as M with two MMAs per k
// step: 0.73 vs 0.91 ms per 26B canvas pass). With few tiles (one canvas) the K loop is
// split over ks independent CTAs on 128-token chunks and the FFN norm that follows adds
// their partials into x (*nparts = ks); otherwise 64-token chunks add into x directly.
cudaError_t o_proj(dllm_handle* h, const LayerW& L, int T, int* nparts) {
  const auto& c = h->c;
  const int d = c.d_model;
  const int kb = c.n_heads * c.head_dim / 64;
  const int tiles128 = (d / 128) * ceil_div(T, 128);
  const int ks = std::min({4, kb, h->num_sms / tiles128});
  *nparts = 0;
  if (ks >= 2 && (long)ks * T * d <= h->opart_elems) {
    EpiPartialT<128> e{h->opart, d, T, (long)T * d};
    DensePartKSched s{d, d / 128, 128, ks};
    *nparts = ks;
    return launch_gemm<128, 4, 1, kSplitB>(h, dim3(tiles128 * ks), L.tm_wo128, h->tm_ao128, kb, 1, s, e, nullptr,
                                           &h->tm_ao128_lo);
  }
  EpiResidualT<64> et{h->x, d, T};
  DenseSched s{d, d / 128, 64};
  return launch_gemm<64, 6, 1, kSplitB>(h, dim3((d / 128) * ceil_div(T, 64)), L.tm_wo128, h->tm_ao64, kb, 1, s, et,
                                        nullptr, &h->tm_ao64_lo);
}

// One grouped gate/up (or down) GEMM over chunks of BN tokens, with MPI weight tiles per
// work item and ACC accumulator buffers (MPI * ACC * 2 * BN TMEM columns <= 512).
template <int BN, int MPI, int ACC>
cudaError_t moe_gate_up(dllm_handle* h, const LayerW& L) {
  const auto& c = h->c;
  const int F = c.ffn_dim, d = c.d_model;
  constexpr int STAGES = (192 * 1024) / (MPI * 16384 + 2 * BN * 128);
  PersistentGroupedSched<MPI> s{h->offsets, h->routed, h->n_routed, h->chunk_prefix, 2 * F, 2 * F / 128,
                                BN};
  EpiSwiGLU<BN> e{h->hbuf, h->hbuf_lo, F};
  return launch_gemm<BN, STAGES, ACC, kSplitB>(h, dim3(h->num_sms), L.tm_wgu, h->tm_xg[BN == 64 ? 2 : 3], d / 64, 1, s, e,
                                               nullptr, &h->tm_xg_lo[BN == 64 ? 2 : 3]);
}

template <int BN, int MPI, int ACC>
cudaError_t moe_down(dllm_handle* h, const LayerW& L) {
  const auto& c = h->c;
  const int F = c.ffn_dim, d = c.d_model;
  constexpr int STAGES = (192 * 1024) / (MPI * 16384 + 2 * BN * 128);
  PersistentGroupedSched<MPI> s{h->offsets, h->routed, h->n_routed, h->chunk_prefix, d, d / 128,
                                BN};
  EpiDown<BN> e{h->obuf, d};
  return launch_gemm<BN, STAGES, ACC, kSplitB>(h, dim3(h->num_sms), L.tm_wd, h->tm_h[BN == 64 ? 2 : 3], F / 64, 1, s, e,
                                               nullptr, &h->tm_h_lo[BN == 64 ? 2 : 3]);
}

// The FP8-weight variants: one weight tile per item; each stage holds the FP8 tile, the
// token chunk and the converted bf16 tile.
template <int BN, int ACC, int STAGES>
cudaError_t moe_gate_up_w8(dllm_handle* h, const LayerW& L) {
  const auto& c = h->c;
  const int F = c.ffn_dim, d = c.d_model;
  PersistentGroupedSched<1, true> s{h->offsets, h->routed, h->n_routed, h->chunk_prefix, 2 * F,
                                    2 * F / 128, BN, L.egu, 1, (F + 127) / 128, (d + 127) / 128};
  EpiSwiGLU<BN> e{h->hbuf, h->hbuf_lo, F};
  return launch_gemm<BN, STAGES, ACC, kSplitB>(h, dim3(h->num_sms), L.tm_wgu8, h->tm_xg[BN == 64 ? 2 : 3], d / 64, 1, s, e,
                                               nullptr, &h->tm_xg_lo[BN == 64 ? 2 : 3], &h->tok_xg);
}

template <int BN, int ACC, int STAGES>
cudaError_t moe_down_w8(dllm_handle* h, const LayerW& L) {
  const auto& c = h->c;
  const int F = c.ffn_dim, d = c.d_model;
  PersistentGroupedSched<1, true> s{h->offsets, h->routed, h->n_routed, h->chunk_prefix, d,
                                    d / 128, BN, L.ed, 0, d / 128, (F + 127) / 128};
  EpiDown<BN> e{h->obuf, d};
  return launch_gemm<BN, STAGES, ACC, kSplitB>(h, dim3(h->num_sms), L.tm_wd8, h->tm_h[BN == 64 ? 2 : 3], F / 64, 1, s, e,
                                               nullptr, &h->tm_h_lo[BN == 64 ? 2 : 3], &h->tok_h);
}

// Grouped expert GEMMs of one layer over chunks of `chunk` tokens (moe_chunk). gate/up:
// one weight tile per item, two accumulator buffers; down at 64-token chunks: two weight
// tiles per item sharing the token chunk (its 22 m tiles leave enough items to spread
// over the SMs), or one with DLLM_MOE_PAIR=0.
cudaError_t moe_gemms(dllm_handle* h, const LayerW& L, int l, int chunk, uint32_t timed) {
  cudaError_t r;
  const bool wide = chunk == 128;
  if ((r = tmark(h, timed, DLLM_TIMING_GATE_UP, l, 0)) != cudaSuccess) return r;
  if (h->w8)
    r = wide ? moe_gate_up_w8<128, 2, 3>(h, L) : moe_gate_up_w8<64, 2, 4>(h, L);
  else
    r = wide ? moe_gate_up<128, 1, 2>(h, L) : moe_gate_up<64, 1, 2>(h, L);
  if (r != cudaSuccess) return r;
  if ((r = tmark(h, timed, DLLM_TIMING_GATE_UP, l, 1)) != cudaSuccess) return r;
  if ((r = tmark(h, timed, DLLM_TIMING_DOWN, l, 0)) != cudaSuccess) return r;
  if (h->w8)
    r = wide ? moe_down_w8<128, 2, 3>(h, L) : moe_down_w8<64, 2, 4>(h, L);
  else if (wide)
    r = moe_down<128, 1, 2>(h, L);
  else
    r = h->moe_pair ? moe_down<64, 2, 2>(h, L) : moe_down<64, 1, 2>(h, L);
  if (r != cudaSuccess) return r;
  return tmark(h, timed, DLLM_TIMING_DOWN, l, 1);
}

// ------------------------------------------------------------------ the pass

int run_layers(dllm_handle* h, int T, int nreq, int tok_per_req, const int* pos0, const int* slot, int causal,
               int splits, bool record, uint32_t timed, const float* final_gain) {
  const auto& c = h->c;
  const int d = c.d_model;
  const int N = T * h->k;
  for (int l = 0; l < c.n_layers; ++l) {
    NvtxRange nvtx_("layer");
    const LayerW& L = h->L[l];
    bf16_t* kc = h->kcache + (size_t)l * h->kv_layer;
    bf16_t* vc = h->vcache + (size_t)l * h->kv_layer;
    if (l == 0) {   // later layers get this norm from the previous layer's combine
      CK(launch_k(h, rmsnorm_kernel, dim3(T), dim3(row_threads(d)), 0, h->x, (const float*)nullptr, 0, 0L,
                  L.attn_norm, d, c.rms_eps, h->y, h->y_lo, h->y_lo2, h->rstd));
      h->launches++;
    }
    CK(tmark(h, timed, DLLM_TIMING_QKV, l, 0));
    CK(qkv_gemm(h, L, kc, vc, T, pos0, slot, tok_per_req));
    CK(tmark(h, timed, DLLM_TIMING_QKV, l, 1));
    CK(tmark(h, timed, DLLM_TIMING_ATTN, l, 0));
    CK(attention(h, kc, vc, T, nreq, tok_per_req, pos0, slot, causal, splits, &L));
    CK(tmark(h, timed, DLLM_TIMING_ATTN, l, 1));
    CK(tmark(h, timed, DLLM_TIMING_OPROJ, l, 0));
    int o_parts = 0;
    CK(o_proj(h, L, T, &o_parts));
    CK(tmark(h, timed, DLLM_TIMING_OPROJ, l, 1));
    CK(tmark(h, timed, DLLM_TIMING_ROUTE, l, 0));
    CK(launch_k(h, rmsnorm_kernel, dim3(T), dim3(row_threads(d)), 0, h->x, (const float*)h->opart, o_parts,
                (long)T * d, L.ffn_norm, d, c.rms_eps, h->y, h->y_lo, (bf16_t*)nullptr, h->rstd));
    h->launches++;
    if (!h->dense) {
      int r_parts = 0;
      if (h->router_tc) {
        CK(router_gemm(h, L, T, &r_parts));
      } else {
        CK(launch_k(h, router_kernel, dim3(ceil_div(T, kRouterTok), ceil_div(h->E, kRouterExp)), dim3(256),
                    kRouterTok * d * sizeof(float), h->x, h->rstd, L.ffn_norm, L.wr, T, d, h->E, h->rlogits));
        h->launches++;
      }
      CK(launch_k(h, topk_kernel, dim3(ceil_div((long)T * 32, 256)), dim3(256), 0, h->rlogits, T, h->E, h->k,
                  h->tk_idx, h->tk_w, (const float*)h->rpart, r_parts, (long)T * h->E));
      h->launches++;
      if (record) {
        CK(cudaMemcpyAsync(h->dbg_logits + (size_t)l * h->T_canvas_max * h->E, h->rlogits,
                           sizeof(float) * T * h->E, cudaMemcpyDeviceToDevice, h->st));
        CK(cudaMemcpyAsync(h->dbg_idx + (size_t)l * h->T_canvas_max * h->k, h->tk_idx, sizeof(int32_t) * T * h->k,
                           cudaMemcpyDeviceToDevice, h->st));
      }
      if (h->force_routing && T == h->force_T) {
        CK(launch_k(h, force_route_kernel, dim3(ceil_div(T, 128)), dim3(128), 0, h->rlogits,
                    h->dbg_force + (size_t)l * h->force_T * h->k, T, h->E, h->k, h->tk_idx, h->tk_w));
        h->launches++;
      }
    } else {
      CK(launch_k(h, dense_route_kernel, dim3(ceil_div(T, 256)), dim3(256), 0, T, h->tk_idx, h->tk_w));
      h->launches++;
    }
    CK(launch_k(h, permute_kernel, dim3(1), dim3(1024), 0, h->tk_idx, N, h->k, h->E, h->offsets, h->slot_of,
                h->row_token, h->routed, h->n_routed, h->chunk_prefix, moe_chunk(N, h->E),
                timed ? h->routed_stat + l : nullptr));
    CK(launch_k(h, gather_rows_kernel, dim3(N), dim3(std::min(1024, (d / 8 + 31) / 32 * 32)), 0, h->y, h->y_lo,
                h->row_token, N, d, h->xg, h->xg_lo));
    h->launches += 2;
    CK(tmark(h, timed, DLLM_TIMING_ROUTE, l, 1));
    CK(moe_gemms(h, L, l, moe_chunk(N, h->E), timed));
    CK(tmark(h, timed, DLLM_TIMING_NORM, l, 0));
    const float* next_gain = l + 1 < c.n_layers ? h->L[l + 1].attn_norm : final_gain;
    // the next layer's attention norm feeds the QKV projection: three bf16 terms
    if (next_gain)
      CK(launch_k(h, combine_norm_kernel, dim3(T), dim3(256), 0, h->x, h->obuf, h->slot_of, h->tk_w, h->k,
                  d, next_gain, c.rms_eps, h->y, h->y_lo, l + 1 < c.n_layers ? h->y_lo2 : (bf16_t*)nullptr));
    else
      CK(launch_k(h, combine_kernel, dim3(T), dim3(256), 0, h->x, h->obuf, h->slot_of, h->tk_w, h->k, d));
    h->launches++;
    CK(tmark(h, timed, DLLM_TIMING_NORM, l, 1));
    if (record)
      CK(cudaMemcpyAsync(h->dbg_xl + (size_t)l * h->T_canvas_max * d, h->x, sizeof(float) * T * d,
                         cudaMemcpyDeviceToDevice, h->st));
  }
  CK(cudaGetLastError());
  return DLLM_OK;
}

// mode 0: denoise pass + commit; mode 1: append pass (K/V of the finished canvas kept).
int run_canvas_pass(dllm_handle* h, int B, int mode) {
  const auto& c = h->c;
  const int C = c.canvas, T = B * C, d = c.d_model;
  const int splits = attn_splits(h, B);
  CK(launch_k(h, embed_kernel, dim3(T), dim3(128), 0, h->emb, h->canvas, mode == 0 ? h->mask : nullptr, c.mask_id, d,
              h->x));
  h->launches++;
  const uint32_t tm = (h->timing && mode == 0) ? h->tmask : 0u;
  int r = run_layers(h, T, B, C, h->d_P, h->d_slot, 0, splits, h->debug && mode == 0,
                     tm, mode == 0 ? h->final_norm : nullptr);
  if (r) return r;
  if (mode == 1) return DLLM_OK;
  if (h->debug) CK(cudaMemcpyAsync(h->dbg_x, h->x, sizeof(float) * T * d, cudaMemcpyDeviceToDevice, h->st));
  CK(tmark(h, tm, DLLM_TIMING_HEAD, 0, 0));   // the final RMSNorm ran in the last layer's combine
  const int nvt = c.vocab / 256;
  {
    EpiLMHead<256> e{h->lm_m, h->lm_s, h->lm_i, nvt, c.mask_id};
    const int mt = ceil_div(T, 128);
    DenseSched s{T, mt, 256};
    CK((launch_gemm<256, 3, 1, kSplitA>(h, dim3(mt * nvt), h->tm_y, h->tm_head, d / 64, 0, s, e, &h->tm_y_lo)));
  }
  CK(launch_k(h, lm_merge_kernel, dim3(ceil_div((long)T * 32, 256)), dim3(256), 0, h->lm_m, h->lm_s, h->lm_i, T, nvt,
              h->conf, h->argmax, (const int*)h->d_err));
  const int threads = ceil_div(C, 32) * 32;
  CK(launch_k(h, commit_kernel, dim3(B), dim3(threads), C * (sizeof(float) + 1), h->canvas, h->mask, h->conf,
              h->argmax, C, h->d_policy, h->d_step, h->d_remaining, nullptr, nullptr,
              (const int*)h->d_err));
  h->launches += 2;
  CK(tmark(h, tm, DLLM_TIMING_HEAD, 0, 1));
  CK(cudaGetLastError());
  return DLLM_OK;
}

int replay_pass(dllm_handle* h, int B, int mode) {
  const int key = B * 2 + mode;
  auto it = h->graphs.find(key);
  if (it == h->graphs.end()) {
    // eager run first: loads modules and sets kernel attributes outside the capture
    long long before = h->launches;
    int r = run_canvas_pass(h, B, mode);
    if (r) return r;
    if (getenv("DLLM_NO_GRAPH")) return DLLM_OK;
    cudaGraph_t g;
    CK(cudaStreamBeginCapture(h->st, cudaStreamCaptureModeRelaxed));
    before = h->launches;
    r = run_canvas_pass(h, B, mode);
    cudaError_t e = cudaStreamEndCapture(h->st, &g);
    if (r) return r;
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaStreamEndCapture");
    Graph gr;
    gr.kernels = h->launches - before;
    h->launches = before;
    e = cudaGraphInstantiate(&gr.exec, g, 0);
    cudaGraphDestroy(g);
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaGraphInstantiate");
    h->graphs[key] = gr;
    return DLLM_OK;   // the eager run above did this call's work; the capture only recorded it
  }
  CK(cudaGraphLaunch(it->second.exec, h->st));
  h->launches += it->second.kernels;
  return DLLM_OK;
}

int check_requests(dllm_handle* h, int B) {
  if (B < 1 || B > h->c.max_batch) return fail(h, DLLM_E_INVAL, "req_count out of range");
  for (int b = 0; b < B; ++b) {
    if (h->P[b] < 0) return fail(h, DLLM_E_STATE, "request slot " + std::to_string(b) + " has no prefill");
    if (h->P[b] + h->c.canvas > h->c.max_ctx) return fail(h, DLLM_E_CTX_FULL, "KV cache full");
  }
  return DLLM_OK;
}

// Device copies of small host state (prefix lengths, slot ids, policy, step counters)
// are written by one-block kernels that take the values as arguments: no host staging
// buffer has to outlive the call, so no call synchronises for them.
int set_ints(dllm_handle* h, int32_t* dst, int n, int v, bool add) {
  CK(launch_k(h, set_ints_kernel, dim3(1), dim3(64), 0, dst, n, v, add ? 1 : 0));
  h->launches++;
  return DLLM_OK;
}

int check_policy(dllm_handle* h, const dllm_policy* p, int max_steps) {
  if (!p) return fail(h, DLLM_E_INVAL, "policy is NULL");
  if (p->kind != DLLM_POLICY_TOPK && p->kind != DLLM_POLICY_THRESHOLD) return fail(h, DLLM_E_INVAL, "policy kind");
  if (p->kind == DLLM_POLICY_TOPK && p->k < 1) return fail(h, DLLM_E_INVAL, "top-k policy needs k >= 1");
  if (max_steps < 1) return fail(h, DLLM_E_INVAL, "max_steps < 1");
  return DLLM_OK;
}

// The policy, and the step counter of requests 0..n_steps-1 (n_steps = 0: counters kept).
int stage_step(dllm_handle* h, const dllm_policy* p, int max_steps, int step, int n_steps) {
  const PolicyDev pd{p->kind == DLLM_POLICY_TOPK ? 0 : 1, p->k, p->tau, p->floor, max_steps, p->t2t ? 1 : 0,
                     p->edit_tau};
  CK(launch_k(h, stage_step_kernel, dim3(1), dim3(64), 0, pd, step, n_steps, h->d_policy, h->d_step));
  h->launches++;
  return DLLM_OK;
}

int check_device_error(dllm_handle* h) {
  int e = 0;
  CK(cudaMemcpy(&e, h->d_err, sizeof(int), cudaMemcpyDeviceToHost));
  if (e != 0) {
    CK(cudaMemset(h->d_err, 0, sizeof(int)));
    return fail(h, DLLM_E_TIMEOUT, "a kernel gave up a bounded wait (code " + std::to_string(e) + ")");
  }
  return DLLM_OK;
}

// After a timed pass over T tokens: adds each grouped GEMM launch's event time and its
// algorithmic bytes (weights of the experts the layer routed to, the token rows read
// and the results written, both at bf16 size).
void accumulate_timing(dllm_handle* h, int T) {
  const int L = h->c.n_layers;
  std::vector<int32_t> nr(L);
  if (cudaMemcpy(nr.data(), h->routed_stat, sizeof(int32_t) * L, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return;
  }
  const double d = h->c.d_model, F = h->c.ffn_dim, N = (double)T * h->k;
  for (int kind = 0; kind < DLLM_TIMING_KINDS; ++kind) {
    if (!(h->tmask & (1u << kind))) continue;
    const int layers = kind == DLLM_TIMING_HEAD ? 1 : L;
    for (int l = 0; l < layers; l += h->tstride) {
      float ms = 0.f;
      const size_t i = ((size_t)kind * L + l) * 2;
      if (cudaEventElapsedTime(&ms, h->tev[i], h->tev[i + 1]) != cudaSuccess) {
        cudaGetLastError();
        continue;
      }
      h->t_ms[kind] += ms;
      h->t_n[kind] += 1;
      // the method's bytes: the routed experts' bf16 weights, the bf16 token rows in and
      // the bf16 results out (the (hi, lo) pairs and fp32 outputs are the kernels' own)
      const double wb = h->w8 ? 1.0 : 2.0;   // weight bytes per element (FP8 or bf16)
      if (kind == DLLM_TIMING_GATE_UP) h->t_bytes[kind] += nr[l] * 2 * F * d * wb + N * d * 2 + N * F * 2;
      if (kind == DLLM_TIMING_DOWN) h->t_bytes[kind] += nr[l] * d * F * wb + N * F * 2 + N * d * 2;
    }
  }
}

void drop_graphs(dllm_handle* h) {
  for (auto& kv : h->graphs)
    if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
  h->graphs.clear();
}

int validate(const dllm_config* c, std::string* why) {
  auto bad = [&](const char* m) { *why = m; return DLLM_E_INVAL; };
  if (c->n_layers < 1 || c->d_model < 256 || c->d_model % 256 || c->d_model > 256 * kRouterMaxChunks)
    return bad("d_model must be a multiple of 256, at most 4096");
  if (c->head_dim != 64 && c->head_dim != 176) return bad("head_dim must be 64 or 176");
  if (c->n_heads < 1 || c->n_kv_heads < 1 || c->n_heads % c->n_kv_heads) return bad("n_heads % n_kv_heads != 0");
  if ((c->n_heads * c->head_dim) % 64) return bad("n_heads * head_dim must be a multiple of 64");
  if (c->ffn_dim < 64 || c->ffn_dim % 64) return bad("ffn_dim must be a multiple of 64");
  if (c->vocab < 256 || c->vocab % 256) return bad("vocab must be a multiple of 256");
  if (c->mask_id != c->vocab - 1) return bad("mask_id must be vocab - 1");
  if (c->n_experts < 0 || c->n_experts > 256) return bad("n_experts in [0, 256]");
  if (c->n_experts == 0 && c->top_k != 1) return bad("dense FFN needs top_k = 1");
  if (c->n_experts > 0 && (c->top_k < 1 || c->top_k > 8 || c->top_k > c->n_experts)) return bad("top_k in [1, 8]");
  if (c->canvas < 1 || c->canvas > 1024) return bad("canvas in [1, 1024]");
  if (c->max_batch < 1 || c->max_ctx < c->canvas + 1) return bad("max_batch >= 1 and max_ctx > canvas");
  if (c->weight_dtype != DLLM_WEIGHTS_F32 && c->weight_dtype != DLLM_WEIGHTS_BF16) return bad("weight_dtype");
  if (c->expert_format != DLLM_EXPERTS_BF16 && c->expert_format != DLLM_EXPERTS_FP8) return bad("expert_format");
  if (c->expert_format == DLLM_EXPERTS_FP8 && c->ffn_dim > 128 * kConvMaxColBlocks)
    return bad("FP8 experts: ffn_dim at most 8192");
  return DLLM_OK;
}

// ------------------------------------------------------------------ weight loading

struct BlobReader {
  const uint8_t* base;
  size_t size;
  size_t off = 0;
  int esize;
  bool on_device;
  const uint8_t* next(size_t numel, bool* ok) {
    size_t o = off;
    size_t bytes = numel * esize;
    if (o + bytes > size) {
      *ok = false;
      return nullptr;
    }
    off = (o + bytes + 255) / 256 * 256;
    return base + o;
  }
};

// Copies one blob tensor into bf16 rows of dst (see pack_rows_kernel for the row map).
int pack_tensor(dllm_handle* h, BlobReader& br, void* staging, bf16_t* dst, long rows, int cols, long group,
                long gstride, long goff) {
  bool ok = true;
  const uint8_t* src = br.next((size_t)rows * cols, &ok);
  if (!ok) return fail(h, DLLM_E_INVAL, "weight blob too small");
  const void* s = src;
  if (!br.on_device) {
    CK(cudaMemcpyAsync(staging, src, (size_t)rows * cols * br.esize, cudaMemcpyHostToDevice, h->st));
    s = staging;
  }
  pack_rows_kernel<<<1184, 256, 0, h->st>>>(dst, s, br.esize == 4, rows, cols, group, gstride, goff);
  CK(cudaGetLastError());
  if (!br.on_device) CK(cudaStreamSynchronize(h->st));
  return DLLM_OK;
}

int load_f32(dllm_handle* h, BlobReader& br, void* staging, float* dst, long n) {
  bool ok = true;
  const uint8_t* src = br.next((size_t)n, &ok);
  if (!ok) return fail(h, DLLM_E_INVAL, "weight blob too small");
  const void* s = src;
  if (!br.on_device) {
    CK(cudaMemcpyAsync(staging, src, (size_t)n * br.esize, cudaMemcpyHostToDevice, h->st));
    s = staging;
  }
  to_f32_kernel<<<64, 256, 0, h->st>>>(dst, s, br.esize == 4, n);
  CK(cudaGetLastError());
  if (!br.on_device) CK(cudaStreamSynchronize(h->st));
  return DLLM_OK;
}

int create_impl(dllm_handle* h, const void* weights, size_t weight_bytes, int on_device) {
  const dllm_config& c = h->c;
  const int d = c.d_model, F = c.ffn_dim, hd = c.head_dim, H = c.n_heads, Hkv = c.n_kv_heads, V = c.vocab;
  h->dense = c.n_experts == 0;
  h->E = h->dense ? 1 : c.n_experts;
  h->k = h->dense ? 1 : c.top_k;
  h->qkv_heads = H + 2 * Hkv;
  {
    int dev = 0;
    CK(cudaGetDevice(&dev));
    CK(cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev));
  }
  // tensor-core attention for canvas passes when a query tile of 128 rows holds whole
  // GQA groups (DLLM_ATTN_LEGACY=1 keeps the warp-MMA kernel, for comparisons)
  h->attn_tc = 128 % (H / Hkv) == 0;
  if (const char* m = getenv("DLLM_MOE_PAIR")) h->moe_pair = atoi(m) != 0;
  h->router_tc = !h->dense && h->E % 32 == 0;
  h->w8 = !h->dense && c.expert_format == DLLM_EXPERTS_FP8;
  const long qd = (long)H * hd, kvd = (long)Hkv * hd;

  // ---- weights
  DA(h->emb, (size_t)V * d);
  DA(h->head, (size_t)V * d);
  DA(h->final_norm, d);
  h->L.resize(c.n_layers);
  for (auto& L : h->L) {
    DA(L.attn_norm, d);
    DA(L.ffn_norm, d);
    DA(L.wqkv, (size_t)(qd + 2 * kvd) * d);
    DA(L.wo, (size_t)d * qd);
    if (!h->dense) DA(L.wr, (size_t)h->E * d);
    if (h->w8) {
      DA(L.wgu8, (size_t)h->E * 2 * F * d);
      DA(L.wd8, (size_t)h->E * d * F);
      DA(L.egu, (size_t)h->E * 2 * ((F + 127) / 128) * ((d + 127) / 128));
      DA(L.ed, (size_t)h->E * (d / 128) * ((F + 127) / 128));
    } else {
      DA(L.wgu, (size_t)h->E * 2 * F * d);
      DA(L.wd, (size_t)h->E * d * F);
    }
  }
  // FP8 experts: each expert matrix is unpacked to bf16 here (original layout), then
  // quantised into its packed FP8 place
  bf16_t* w8_src = nullptr;
  if (h->w8) DA(w8_src, (size_t)F * d);
  uint8_t* staging = nullptr;
  if (!on_device) {
    const size_t sizes[] = {(size_t)V * d, (size_t)qd * d, (size_t)kvd * d, (size_t)F * d, (size_t)h->E * d};
    size_t mx = 0;   // elements of the largest blob tensor
    for (size_t s : sizes) mx = s > mx ? s : mx;
    DA(staging, mx * 4 + 256);   // bytes, fp32 worst case
  }
  BlobReader br{reinterpret_cast<const uint8_t*>(weights), weight_bytes, 0,
                c.weight_dtype == DLLM_WEIGHTS_F32 ? 4 : 2, on_device != 0};
  const long BIG = 1L << 40;
  int r;
  if ((r = pack_tensor(h, br, staging, h->emb, V, d, BIG, 0, 0))) return r;
  for (int l = 0; l < c.n_layers; ++l) {
    LayerW& L = h->L[l];
    if ((r = load_f32(h, br, staging, L.attn_norm, d))) return r;
    if ((r = pack_tensor(h, br, staging, L.wqkv, qd, d, BIG, 0, 0))) return r;
    if ((r = pack_tensor(h, br, staging, L.wqkv, kvd, d, BIG, 0, qd))) return r;
    if ((r = pack_tensor(h, br, staging, L.wqkv, kvd, d, BIG, 0, qd + kvd))) return r;
    if ((r = pack_tensor(h, br, staging, L.wo, d, (int)qd, BIG, 0, 0))) return r;
    if ((r = load_f32(h, br, staging, L.ffn_norm, d))) return r;
    if (!h->dense)
      if ((r = pack_tensor(h, br, staging, L.wr, h->E, d, BIG, 0, 0))) return r;
    for (int e = 0; e < h->E; ++e) {
      const long gu0 = (long)e * 2 * F;
      if (h->w8) {
        const int nrbF = (F + 127) / 128, ncbD = (d + 127) / 128, nrbD = d / 128, ncbF = (F + 127) / 128;
        for (int which = 0; which < 2; ++which) {   // gate rows, then up rows
          if ((r = pack_tensor(h, br, staging, w8_src, F, d, BIG, 0, 0))) return r;
          CK(launch_k(h, quantize_e4m3_blocks_kernel, dim3(ncbD, nrbF), dim3(256), 0, w8_src, F, d, L.wgu8,
                      L.egu + (size_t)(e * 2 + which) * nrbF * ncbD, 64L, 128L, gu0 + 64 * which));
        }
        if ((r = pack_tensor(h, br, staging, w8_src, d, F, BIG, 0, 0))) return r;
        CK(launch_k(h, quantize_e4m3_blocks_kernel, dim3(ncbF, nrbD), dim3(256), 0, w8_src, d, F, L.wd8,
                    L.ed + (size_t)e * nrbD * ncbF, BIG, 0L, (long)e * d));
        continue;
      }
      if ((r = pack_tensor(h, br, staging, L.wgu, F, d, 64, 128, gu0))) return r;        // gate rows
      if ((r = pack_tensor(h, br, staging, L.wgu, F, d, 64, 128, gu0 + 64))) return r;   // up rows
      if ((r = pack_tensor(h, br, staging, L.wd, d, F, BIG, 0, (long)e * d))) return r;
    }
  }
  if ((r = load_f32(h, br, staging, h->final_norm, d))) return r;
  if ((r = pack_tensor(h, br, staging, h->head, V, d, BIG, 0, 0))) return r;

  // ---- RoPE tables (fp64 on the host, stored fp32)
  const int half = hd / 2;
  {
    std::vector<float> cs((size_t)c.max_ctx * half), sn((size_t)c.max_ctx * half);
    for (int p = 0; p < c.max_ctx; ++p)
      for (int i = 0; i < half; ++i) {
        const double inv = pow((double)c.rope_theta, -2.0 * i / hd);
        const double a = (double)p * inv;
        cs[(size_t)p * half + i] = (float)cos(a);
        sn[(size_t)p * half + i] = (float)sin(a);
      }
    DA(h->rope_cos, cs.size());
    DA(h->rope_sin, sn.size());
    CK(cudaMemcpy(h->rope_cos, cs.data(), cs.size() * 4, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(h->rope_sin, sn.data(), sn.size() * 4, cudaMemcpyHostToDevice));
  }

  // ---- KV cache
  h->kv_layer = (size_t)c.max_batch * Hkv * c.max_ctx * hd;
  DA(h->kcache, h->kv_layer * c.n_layers);
  DA(h->vcache, h->kv_layer * c.n_layers);
  CK(cudaMemsetAsync(h->kcache, 0, h->kv_layer * c.n_layers * 2, h->st));
  CK(cudaMemsetAsync(h->vcache, 0, h->kv_layer * c.n_layers * 2, h->st));

  // ---- activations
  h->T_canvas_max = c.max_batch * c.canvas;
  h->T_max = h->T_canvas_max > c.max_ctx - c.canvas ? h->T_canvas_max : c.max_ctx - c.canvas;
  h->N_max = h->T_max * h->k;
  const int T = h->T_max, N = h->N_max;
  DA(h->x, (size_t)T * d);
  DA(h->y, (size_t)T * d);
  DA(h->y_lo, (size_t)T * d);
  DA(h->y_lo2, (size_t)T * d);
  DA(h->rstd, T);
  DA(h->q, (size_t)T * qd);
  DA(h->ao, (size_t)T * qd);
  DA(h->ao_lo, (size_t)T * qd);
  {
    size_t mx = 0;
    for (int B = 1; B <= c.max_batch; ++B) {
      const int s = attn_splits(h, B);
      if (s > 1 && (size_t)s * B > mx) mx = (size_t)s * B;
    }
    DA(h->apart, mx * c.canvas * qd + 1);
    DA(h->alse, mx * c.canvas * H + 1);
  }
  DA(h->rlogits, (size_t)T * h->E);
  // split-K partials exist only while slices x tiles <= 2 x the SM count (router:
  // 32-expert tiles of 128 rows) or <= the SM count (O projection: 128 x 128 tiles),
  // which bounds their size
  h->rpart_elems = 2L * h->num_sms * 128 * 32;
  h->opart_elems = (long)h->num_sms * 128 * 128;
  DA(h->rpart, (size_t)h->rpart_elems);
  DA(h->opart, (size_t)h->opart_elems);
  DA(h->tk_idx, (size_t)N);
  DA(h->tk_w, (size_t)N);
  DA(h->offsets, h->E + 1);
  DA(h->routed, h->E);
  DA(h->n_routed, 1);
  DA(h->chunk_prefix, h->E + 1);
  DA(h->routed_stat, c.n_layers);

  DA(h->slot_of, (size_t)N);
  DA(h->row_token, (size_t)N);
  DA(h->xg, (size_t)N * d);
  DA(h->xg_lo, (size_t)N * d);
  DA(h->hbuf, (size_t)N * F);
  DA(h->hbuf_lo, (size_t)N * F);
  DA(h->obuf, (size_t)N * d);
  const int nvt = V / 256;
  DA(h->lm_m, (size_t)h->T_canvas_max * nvt);
  DA(h->lm_s, (size_t)h->T_canvas_max * nvt);
  DA(h->lm_i, (size_t)h->T_canvas_max * nvt);
  DA(h->conf, h->T_canvas_max);
  DA(h->argmax, h->T_canvas_max);
  CK(cudaMemsetAsync(h->q, 0, (size_t)T * qd * 2, h->st));   // padding rows of a query tile read zeros
  CK(cudaMemsetAsync(h->xg, 0, (size_t)N * d * 2, h->st));
  CK(cudaMemsetAsync(h->xg_lo, 0, (size_t)N * d * 2, h->st));
  CK(cudaMemsetAsync(h->hbuf, 0, (size_t)N * F * 2, h->st));
  CK(cudaMemsetAsync(h->hbuf_lo, 0, (size_t)N * F * 2, h->st));

  // ---- request state
  h->P.assign(c.max_batch, -1);
  h->passed.assign(c.max_batch, 0);
  DA(h->d_P, c.max_batch);
  DA(h->d_slot, c.max_batch);
  DA(h->d_pre_pos, 1);
  DA(h->d_pre_slot, 1);
  DA(h->d_tokens, T);
  DA(h->canvas, h->T_canvas_max);
  DA(h->mask, h->T_canvas_max);
  DA(h->d_step, c.max_batch);
  DA(h->d_remaining, c.max_batch);
  DA(h->d_policy, 1);
  DA(h->d_err, 1);
  {
    std::vector<int32_t> s(c.max_batch);
    for (int i = 0; i < c.max_batch; ++i) s[i] = i;
    CK(cudaMemcpy(h->d_slot, s.data(), sizeof(int32_t) * s.size(), cudaMemcpyHostToDevice));
  }
  CK(cudaMemset(h->d_pre_pos, 0, sizeof(int32_t)));
  CK(cudaMemset(h->d_err, 0, sizeof(int)));
  CK(cudaMemset(h->d_P, 0, sizeof(int32_t) * c.max_batch));
  CK(cudaMallocHost(&h->h_remaining, sizeof(int32_t) * c.max_batch));

  // ---- tensor maps
  bool ok = true;
  ok &= make_tmap(&h->tm_y, h->y, T, d, 128);
  ok &= make_tmap(&h->tm_y_lo, h->y_lo, T, d, 128);
  ok &= make_tmap(&h->tm_y_lo2, h->y_lo2, T, d, 128);
  ok &= make_tmap(&h->tm_ao64, h->ao, T, qd, 64);
  ok &= make_tmap(&h->tm_ao64_lo, h->ao_lo, T, qd, 64);
  ok &= make_tmap(&h->tm_ao128, h->ao, T, qd, 128);
  ok &= make_tmap(&h->tm_ao128_lo, h->ao_lo, T, qd, 128);
  ok &= make_tmap(&h->tm_head, h->head, V, d, 256);
  if (h->attn_tc) ok &= make_tmap3(&h->tm_q3, h->q, hd, H, T, H / Hkv, 128 / (H / Hkv));
  for (int i = 0; i < 4; ++i) {
    ok &= make_tmap(&h->tm_xg[i], h->xg, N, d, kMoeBN[i]);
    ok &= make_tmap(&h->tm_xg_lo[i], h->xg_lo, N, d, kMoeBN[i]);
    ok &= make_tmap(&h->tm_h[i], h->hbuf, N, F, kMoeBN[i]);
    ok &= make_tmap(&h->tm_h_lo[i], h->hbuf_lo, N, F, kMoeBN[i]);
  }
  for (auto& L : h->L) {
    ok &= make_tmap(&L.tm_wqkv, L.wqkv, qd + 2 * kvd, d, hd);
    ok &= make_tmap(&L.tm_wo, L.wo, d, qd, 64);
    ok &= make_tmap(&L.tm_wo128, L.wo, d, qd, 128);
    if (h->router_tc) ok &= make_tmap(&L.tm_wr, L.wr, h->E, d, 32);
    if (h->w8) {
      ok &= make_tmap_u8(&L.tm_wgu8, L.wgu8, (uint64_t)h->E * 2 * F, d, 128);
      ok &= make_tmap_u8(&L.tm_wd8, L.wd8, (uint64_t)h->E * d, F, 128);
    } else {
      ok &= make_tmap(&L.tm_wgu, L.wgu, (uint64_t)h->E * 2 * F, d, 128);
      ok &= make_tmap(&L.tm_wd, L.wd, (uint64_t)h->E * d, F, 128);
    }
    if (h->attn_tc) {
      const size_t l = &L - h->L.data();
      const uint64_t kv_rows = (uint64_t)c.max_batch * Hkv * c.max_ctx;
      ok &= make_tmap(&L.tm_k, h->kcache + l * h->kv_layer, kv_rows, hd, 64);
      ok &= make_tmap(&L.tm_v, h->vcache + l * h->kv_layer, kv_rows, hd, 64);
    }
  }
  if (!ok) return fail(h, DLLM_E_CUDA, "cuTensorMapEncodeTiled failed");
  for (int i = 0; i < 4; ++i) {
    h->tok_xg.m[i] = h->tm_xg[i];
    h->tok_xg.m[4 + i] = h->tm_xg_lo[i];
    h->tok_h.m[i] = h->tm_h[i];
    h->tok_h.m[4 + i] = h->tm_h_lo[i];
  }
  CK(cudaFuncSetAttribute(reinterpret_cast<const void*>(router_kernel), cudaFuncAttributeMaxDynamicSharedMemorySize,
                          kRouterTok * d * (int)sizeof(float)));
  CK(cudaStreamSynchronize(h->st));
  return DLLM_OK;
}

void free_all(dllm_handle* h) {
  drop_graphs(h);
  for (auto& e : h->tev) cudaEventDestroy(e);
  h->tev.clear();
  for (void* p : h->allocs) cudaFree(p);
  h->allocs.clear();
  if (h->h_remaining) cudaFreeHost(h->h_remaining);
  h->h_remaining = nullptr;
  if (h->own_stream && h->st) cudaStreamDestroy(h->st);
  h->st = nullptr;
}

int prefill_impl(dllm_handle* h, int req, const int32_t* prompt, int n, bool prompt_on_host) {
  const auto& c = h->c;
  if (req < 0 || req >= c.max_batch) return fail(h, DLLM_E_INVAL, "req out of range");
  if (n < 1 || !prompt) return fail(h, DLLM_E_INVAL, "empty prompt");
  if (n + c.canvas > c.max_ctx) return fail(h, DLLM_E_CTX_FULL, "prompt + canvas exceeds max_ctx");
  CK(cudaMemcpyAsync(h->d_tokens, prompt, sizeof(int32_t) * n,
                     prompt_on_host ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToDevice, h->st));
  int r = set_ints(h, h->d_pre_slot, 1, req, false);
  if (r) return r;
  CK(launch_k(h, embed_kernel, dim3(n), dim3(128), 0, h->emb, h->d_tokens, nullptr, c.mask_id, c.d_model, h->x));
  h->launches++;
  r = run_layers(h, n, 1, n, h->d_pre_pos, h->d_pre_slot, 1, 1, false, 0u, nullptr);
  if (r) return r;
  h->P[req] = n;
  h->passed[req] = 0;
  return set_ints(h, h->d_P + req, 1, n, false);
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

int dllm_create(const dllm_config* cfg, const void* weights, size_t weight_bytes, int weights_on_device,
                void* cuda_stream, dllm_handle** out) {
  if (!out) return DLLM_E_INVAL;
  *out = nullptr;
  if (!cfg || !weights) return DLLM_E_INVAL;
  std::string why;
  if (validate(cfg, &why)) {
    fprintf(stderr, "dllm_create: %s\n", why.c_str());
    return DLLM_E_INVAL;
  }
  dllm_handle* h = new dllm_handle();
  h->c = *cfg;
  if (cuda_stream) {
    h->st = reinterpret_cast<cudaStream_t>(cuda_stream);
  } else {
    if (cudaStreamCreateWithFlags(&h->st, cudaStreamNonBlocking) != cudaSuccess) {
      delete h;
      return DLLM_E_CUDA;
    }
    h->own_stream = true;
  }
  int r = create_impl(h, weights, weight_bytes, weights_on_device);
  if (r) {
    fprintf(stderr, "dllm_create: %s\n", h->err.c_str());
    free_all(h);
    delete h;
    return r;
  }
  *out = h;
  return DLLM_OK;
}

int dllm_prefill(dllm_handle* h, int req, const int32_t* prompt, int n) {
  if (!h) return DLLM_E_INVAL;
  NvtxRange nvtx_("dllm_prefill");
  return prefill_impl(h, req, prompt, n, false);
}

int dllm_denoise_step(dllm_handle* h, int req_count, int32_t* canvas, uint8_t* mask, const dllm_policy* policy,
                      int step, int max_steps, float* conf_out, int32_t* argmax_out, int32_t* remaining_out) {
  if (!h) return DLLM_E_INVAL;
  NvtxRange nvtx_("dllm_denoise_step");
  if (!canvas || !mask) return fail(h, DLLM_E_INVAL, "canvas/mask NULL");
  int r = check_requests(h, req_count);
  if (r) return r;
  if (step < 0) return fail(h, DLLM_E_INVAL, "step < 0");
  if ((r = check_policy(h, policy, max_steps))) return r;
  const int C = h->c.canvas, B = req_count;
  if ((r = stage_step(h, policy, max_steps, step, B))) return r;
  CK(cudaMemcpyAsync(h->canvas, canvas, sizeof(int32_t) * B * C, cudaMemcpyDeviceToDevice, h->st));
  CK(cudaMemcpyAsync(h->mask, mask, (size_t)B * C, cudaMemcpyDeviceToDevice, h->st));
  if ((r = replay_pass(h, B, 0))) return r;
  h->last_B = B;
  for (int b = 0; b < B; ++b) h->passed[b] = 1;
  CK(cudaMemcpyAsync(canvas, h->canvas, sizeof(int32_t) * B * C, cudaMemcpyDeviceToDevice, h->st));
  CK(cudaMemcpyAsync(mask, h->mask, (size_t)B * C, cudaMemcpyDeviceToDevice, h->st));
  if (conf_out) CK(cudaMemcpyAsync(conf_out, h->conf, sizeof(float) * B * C, cudaMemcpyDeviceToDevice, h->st));
  if (argmax_out)
    CK(cudaMemcpyAsync(argmax_out, h->argmax, sizeof(int32_t) * B * C, cudaMemcpyDeviceToDevice, h->st));
  if (remaining_out)
    CK(cudaMemcpyAsync(remaining_out, h->d_remaining, sizeof(int32_t) * B, cudaMemcpyDeviceToDevice, h->st));
  return DLLM_OK;
}

int dllm_generate_block(dllm_handle* h, int req_count, int max_steps, const dllm_policy* policy, int32_t* canvas_out,
                        int* steps_taken) {
  if (!h) return DLLM_E_INVAL;
  NvtxRange nvtx_("dllm_generate_block");
  int r = check_requests(h, req_count);
  if (r) return r;
  if ((r = check_policy(h, policy, max_steps))) return r;
  const int C = h->c.canvas, B = req_count;
  if ((r = stage_step(h, policy, max_steps, 0, 0))) return r;
  CK(launch_k(h, canvas_init_kernel, dim3(ceil_div((long)B * C, 256)), dim3(256), 0, h->canvas, h->mask, B * C,
              h->c.mask_id, h->d_step, B));
  h->launches++;
  std::vector<int> done_at(B, -1);
  int s = 0;
  bool all_done = false;
  for (; s < max_steps && !all_done; ++s) {
    if ((r = replay_pass(h, B, 0))) return r;
    for (int b = 0; b < B; ++b) h->passed[b] = 1;
    CK(cudaMemcpyAsync(h->h_remaining, h->d_remaining, sizeof(int32_t) * B, cudaMemcpyDeviceToHost, h->st));
    CK(cudaStreamSynchronize(h->st));
    if (h->timing) accumulate_timing(h, B * C);
    all_done = true;
    bool aborted = false;
    for (int b = 0; b < B; ++b) {
      if (h->h_remaining[b] == 0 && done_at[b] < 0) done_at[b] = s + 1;
      if (h->h_remaining[b] != 0) all_done = false;
      if (h->h_remaining[b] < 0) aborted = true;   // a kernel of the pass gave up a bounded wait
    }
    if (aborted) {
      ++s;
      break;
    }
  }
  h->last_B = B;
  if ((r = check_device_error(h))) return r;
  if (steps_taken)
    for (int b = 0; b < B; ++b) steps_taken[b] = done_at[b] < 0 ? s : done_at[b];
  if (canvas_out)
    CK(cudaMemcpyAsync(canvas_out, h->canvas, sizeof(int32_t) * B * C, cudaMemcpyDeviceToDevice, h->st));
  if (!all_done) return fail(h, DLLM_E_BUDGET, "step budget spent with masked positions left");
  return DLLM_OK;
}

int dllm_append_kv(dllm_handle* h, int req_count, const int32_t* canvas) {
  if (!h) return DLLM_E_INVAL;
  NvtxRange nvtx_("dllm_append_kv");
  int r = check_requests(h, req_count);
  if (r) return r;
  const int C = h->c.canvas, B = req_count;
  if (canvas) CK(cudaMemcpyAsync(h->canvas, canvas, sizeof(int32_t) * B * C, cudaMemcpyDeviceToDevice, h->st));
  if ((r = replay_pass(h, B, 1))) return r;
  for (int b = 0; b < B; ++b) {
    h->P[b] += C;
    h->passed[b] = 0;
  }
  return set_ints(h, h->d_P, B, C, true);
}

int dllm_append_kv_approx(dllm_handle* h, int req_count) {
  if (!h) return DLLM_E_INVAL;
  NvtxRange nvtx_("dllm_append_kv_approx");
  int r = check_requests(h, req_count);
  if (r) return r;
  for (int b = 0; b < req_count; ++b)
    if (!h->passed[b]) return fail(h, DLLM_E_STATE, "slot " + std::to_string(b) + " has no canvas pass to keep");
  // the K/V that the last canvas pass wrote at P..P+C-1 stay where they are
  for (int b = 0; b < req_count; ++b) {
    h->P[b] += h->c.canvas;
    h->passed[b] = 0;
  }
  return set_ints(h, h->d_P, req_count, h->c.canvas, true);
}

int dllm_generate(dllm_handle* h, int req_count, const int32_t* prompts, int n_prompt, int n_canvases, int max_steps,
                  const dllm_policy* policy, int32_t* tokens_out, int* steps_out) {
  if (!h) return DLLM_E_INVAL;
  NvtxRange nvtx_("dllm_generate");
  if (!prompts || !tokens_out || n_canvases < 1) return fail(h, DLLM_E_INVAL, "bad arguments");
  if (req_count < 1 || req_count > h->c.max_batch) return fail(h, DLLM_E_INVAL, "req_count out of range");
  const int C = h->c.canvas;
  if (n_prompt + (long)n_canvases * C + C > (long)h->c.max_ctx + C)
    return fail(h, DLLM_E_CTX_FULL, "prompt + canvases exceed max_ctx");
  int r;
  for (int b = 0; b < req_count; ++b)
    if ((r = prefill_impl(h, b, prompts + (size_t)b * n_prompt, n_prompt, true))) return r;
  std::vector<int> steps(req_count);
  for (int ci = 0; ci < n_canvases; ++ci) {
    if ((r = dllm_generate_block(h, req_count, max_steps, policy, nullptr, steps.data()))) return r;
    for (int b = 0; b < req_count; ++b) {
      CK(cudaMemcpyAsync(tokens_out + ((size_t)b * n_canvases + ci) * C, h->canvas + (size_t)b * C,
                         sizeof(int32_t) * C, cudaMemcpyDeviceToHost, h->st));
      if (steps_out) steps_out[(size_t)b * n_canvases + ci] = steps[b];
    }
    if ((r = dllm_append_kv(h, req_count, nullptr))) return r;
  }
  CK(cudaStreamSynchronize(h->st));
  return check_device_error(h);
}

int dllm_reset(dllm_handle* h, int req) {
  if (!h) return DLLM_E_INVAL;
  if (req < 0 || req >= h->c.max_batch) return fail(h, DLLM_E_INVAL, "req out of range");
  h->P[req] = -1;
  h->passed[req] = 0;
  return set_ints(h, h->d_P + req, 1, 0, false);
}

int dllm_prefix_len(const dllm_handle* h, int req) {
  if (!h || req < 0 || req >= h->c.max_batch) return DLLM_E_INVAL;
  return h->P[req] < 0 ? 0 : h->P[req];
}

int dllm_check(dllm_handle* h) {
  if (!h) return DLLM_E_INVAL;
  CK(cudaStreamSynchronize(h->st));
  CK(cudaGetLastError());
  return check_device_error(h);
}

long long dllm_launch_count(const dllm_handle* h) { return h ? h->launches : -1; }

int dllm_set_wait_limit(dllm_handle* h, long long ns) {
  if (!h) return DLLM_E_INVAL;
  const unsigned long long v = ns > 0 ? (unsigned long long)ns : kWaitLimitNs;
  CK(cudaStreamSynchronize(h->st));
  CK(cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)));
  return DLLM_OK;
}

int dllm_set_debug(dllm_handle* h, int on) {
  if (!h) return DLLM_E_INVAL;
  if (on && !h->dbg_x) {
    const size_t T = h->T_canvas_max;
    DA(h->dbg_logits, (size_t)h->c.n_layers * T * h->E);
    DA(h->dbg_idx, (size_t)h->c.n_layers * T * h->k);
    DA(h->dbg_x, T * h->c.d_model);
    DA(h->dbg_xl, (size_t)h->c.n_layers * T * h->c.d_model);
  }
  h->debug = on != 0;
  drop_graphs(h);
  return DLLM_OK;
}

int dllm_debug_force_routing(dllm_handle* h, const int32_t* idx, int T) {
  if (!h) return DLLM_E_INVAL;
  if (!h->debug) return fail(h, DLLM_E_STATE, "debug is off");
  if (h->dense) return fail(h, DLLM_E_INVAL, "dense model has no routing");
  drop_graphs(h);
  if (!idx) {
    h->force_routing = false;
    return DLLM_OK;
  }
  if (T < 1 || T > h->T_max) return fail(h, DLLM_E_INVAL, "T out of range");
  const size_t n = (size_t)h->c.n_layers * T * h->k;
  for (size_t i = 0; i < n; ++i)
    if (idx[i] < 0 || idx[i] >= h->E) return fail(h, DLLM_E_INVAL, "expert index out of range");
  if (!h->dbg_force) DA(h->dbg_force, (size_t)h->c.n_layers * h->T_max * h->k);
  CK(cudaMemcpy(h->dbg_force, idx, sizeof(int32_t) * n, cudaMemcpyHostToDevice));
  h->force_T = T;
  h->force_routing = true;
  return DLLM_OK;
}

int dllm_debug_read(dllm_handle* h, int what, int layer, void* dst, size_t bytes) {
  if (!h || !dst) return DLLM_E_INVAL;
  if (!h->debug) return fail(h, DLLM_E_STATE, "debug is off");
  const size_t T = (size_t)h->last_B * h->c.canvas;
  const void* src = nullptr;
  size_t need = 0;
  if (layer < 0 || layer >= h->c.n_layers) layer = 0;
  switch (what) {
    case 0: src = h->dbg_x; need = T * h->c.d_model * 4; break;
    case 1: src = h->dbg_logits + (size_t)layer * h->T_canvas_max * h->E; need = T * h->E * 4; break;
    case 2: src = h->dbg_idx + (size_t)layer * h->T_canvas_max * h->k; need = T * h->k * 4; break;
    case 3: src = h->conf; need = T * 4; break;
    case 4: src = h->argmax; need = T * 4; break;
    case 5: src = h->dbg_xl + (size_t)layer * h->T_canvas_max * h->c.d_model; need = T * h->c.d_model * 4; break;
    case 6:   // K cache of `layer`, slot 0: [Hkv][max_ctx][hd] bf16
      src = h->kcache + (size_t)layer * h->kv_layer;
      need = (size_t)h->c.n_kv_heads * h->c.max_ctx * h->c.head_dim * 2;
      break;
    case 7:   // V cache of `layer`, slot 0
      src = h->vcache + (size_t)layer * h->kv_layer;
      need = (size_t)h->c.n_kv_heads * h->c.max_ctx * h->c.head_dim * 2;
      break;
    default: return fail(h, DLLM_E_INVAL, "unknown debug buffer");
  }
  if (bytes < need) return fail(h, DLLM_E_INVAL, "debug buffer too small");
  CK(cudaStreamSynchronize(h->st));
  CK(cudaMemcpy(dst, src, need, cudaMemcpyDeviceToHost));
  return DLLM_OK;
}

int dllm_set_timing(dllm_handle* h, int kinds) {
  if (!h) return DLLM_E_INVAL;
  if (kinds && h->tev.empty()) {
    h->tev.resize((size_t)DLLM_TIMING_KINDS * h->c.n_layers * 2);
    for (auto& e : h->tev) CK(cudaEventCreate(&e));
  }
  h->tmask = (uint32_t)kinds & ((1u << DLLM_TIMING_KINDS) - 1);
  const int stride = ((uint32_t)kinds >> DLLM_TIMING_STRIDE_SHIFT) & 0xFF;
  h->tstride = stride > 0 ? stride : 1;
  h->timing = h->tmask != 0;
  drop_graphs(h);
  return DLLM_OK;
}

int dllm_timing_read(dllm_handle* h, double* total_ms, long long* launches, double* bytes, int reset) {
  if (!h || !total_ms || !launches || !bytes) return DLLM_E_INVAL;
  for (int k = 0; k < DLLM_TIMING_KINDS; ++k) {
    total_ms[k] = h->t_ms[k];
    launches[k] = h->t_n[k];
    bytes[k] = h->t_bytes[k];
    if (reset) {
      h->t_ms[k] = 0;
      h->t_n[k] = 0;
      h->t_bytes[k] = 0;
    }
  }
  return DLLM_OK;
}

const char* dllm_last_error(const dllm_handle* h) { return h ? h->err.c_str() : "null handle"; }

void dllm_destroy(dllm_handle* h) {
  if (!h) return;
  if (h->st) cudaStreamSynchronize(h->st);
  free_all(h);
  delete h;
}

// ---------------------------------------------------------------- single-operation entry points

int dllm_op_gemm_bf16(const uint16_t* A, const uint16_t* B, float* D, int M, int N, int K, void* stream) {
  if (!A || !B || !D || M < 1 || N < 128 || N % 128 || K < 64 || K % 64) return DLLM_E_INVAL;
  dllm_handle tmp;
  tmp.st = reinterpret_cast<cudaStream_t>(stream);
  dllm_handle* h = &tmp;
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, A, M, K, 128) || !make_tmap(&tb, B, N, K, 128)) return DLLM_E_INVAL;
  int* err = nullptr;
  CK(cudaMallocAsync(reinterpret_cast<void**>(&err), sizeof(int), tmp.st));
  CK(cudaMemsetAsync(err, 0, sizeof(int), tmp.st));
  tmp.d_err = err;
  const int mt = ceil_div(M, 128);
  DenseSched s{M, mt, 128};
  EpiStoreF32<128> e{D, N, N};
  cudaError_t r = launch_gemm<128, 4, 1, kSplitNone>(h, dim3(mt * (N / 128)), ta, tb, K / 64, 0, s, e);
  if (r == cudaSuccess) {
    poison_on_error_kernel<<<148, 256, 0, tmp.st>>>(err, D, (long)M * N);
    r = cudaGetLastError();
  }
  cudaFreeAsync(err, tmp.st);
  tmp.d_err = nullptr;
  if (r != cudaSuccess) return DLLM_E_CUDA;
  return DLLM_OK;
}

int dllm_op_lm_head_conf(const uint16_t* y, const uint16_t* head, int T, int d, int V, int mask_id, float* conf,
                         int32_t* argmax, void* stream) {
  if (!y || !head || !conf || !argmax || T < 1 || d < 64 || d % 64 || V < 256 || V % 256) return DLLM_E_INVAL;
  dllm_handle tmp;
  tmp.st = reinterpret_cast<cudaStream_t>(stream);
  dllm_handle* h = &tmp;
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, y, T, d, 128) || !make_tmap(&tb, head, V, d, 256)) return DLLM_E_INVAL;
  const int nvt = V / 256;
  float *pm = nullptr, *ps = nullptr;
  int32_t* pi = nullptr;
  int* err = nullptr;
  CK(cudaMallocAsync(reinterpret_cast<void**>(&pm), sizeof(float) * T * nvt, tmp.st));
  CK(cudaMallocAsync(reinterpret_cast<void**>(&ps), sizeof(float) * T * nvt, tmp.st));
  CK(cudaMallocAsync(reinterpret_cast<void**>(&pi), sizeof(int32_t) * T * nvt, tmp.st));
  CK(cudaMallocAsync(reinterpret_cast<void**>(&err), sizeof(int), tmp.st));
  CK(cudaMemsetAsync(err, 0, sizeof(int), tmp.st));
  tmp.d_err = err;
  const int mt = ceil_div(T, 128);
  DenseSched s{T, mt, 256};
  EpiLMHead<256> e{pm, ps, pi, nvt, mask_id};
  cudaError_t r = launch_gemm<256, 4, 1, kSplitNone>(h, dim3(mt * nvt), ta, tb, d / 64, 0, s, e);
  if (r == cudaSuccess) {
    lm_merge_kernel<<<ceil_div((long)T * 32, 256), 256, 0, tmp.st>>>(pm, ps, pi, T, nvt, conf, argmax, err);
    r = cudaGetLastError();
  }
  cudaFreeAsync(pm, tmp.st);
  cudaFreeAsync(ps, tmp.st);
  cudaFreeAsync(pi, tmp.st);
  cudaFreeAsync(err, tmp.st);
  tmp.d_err = nullptr;
  return r == cudaSuccess ? DLLM_OK : DLLM_E_CUDA;
}

int dllm_op_quantize_fp8(const uint16_t* w, int rows, int cols, uint8_t* q, int8_t* exps, void* stream) {
  if (!w || !q || !exps || rows < 1 || cols < 16 || cols % 16) return DLLM_E_INVAL;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  quantize_e4m3_blocks_kernel<<<dim3((cols + 127) / 128, (rows + 127) / 128), 256, 0, st>>>(
      w, rows, cols, q, exps, 1L << 40, 0L, 0L);
  return cudaGetLastError() == cudaSuccess ? DLLM_OK : DLLM_E_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------- allocation-free LM head
//
// The same fused LM head as dllm_op_lm_head_conf, for callers that cannot allocate
// device memory at call time: processes whose device memory is reserved up front under
// a fixed budget (a serving host that hands the whole device to its own allocator and
// refuses foreign cudaMalloc calls), or code paths where an allocation's implicit
// synchronisation or possible failure is not acceptable. Its scratch (the per-row,
// per-vocabulary-tile partials and the error word) lives in one fixed device array in
// this file instead: every GPU that loads the library holds it, 3 MiB plus a few bytes,
// until the process exits.

namespace {

constexpr int kNoAllocMaxRows = 1024;    // rows T per call
constexpr int kNoAllocMaxTiles = 256;    // vocabulary tiles of 256: V <= 65536
constexpr size_t kNoAllocPartials = (size_t)kNoAllocMaxRows * kNoAllocMaxTiles;
// layout: m[partials] fp32 | s[partials] fp32 | idx[partials] int32 | error word (+ pad)
constexpr size_t kNoAllocBytes = kNoAllocPartials * 12 + 256;

// Host code sees only a stand-in for this name; the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoAllocMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device.
cudaError_t noalloc_scratch(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = p;
  }
  *out = reinterpret_cast<unsigned char*>(g_noalloc_addr[dev]);
  return cudaSuccess;
}

}  // namespace

extern "C" int dllm_op_lm_head_conf_noalloc(const uint16_t* y, const uint16_t* head, int T, int d, int V,
                                            int mask_id, float* conf, int32_t* argmax, void* stream) {
  if (!y || !head || !conf || !argmax || T < 1 || d < 64 || d % 64 || V < 256 || V % 256) return DLLM_E_INVAL;
  if (T > kNoAllocMaxRows || V / 256 > kNoAllocMaxTiles) {
    fprintf(stderr,
            "dllm_op_lm_head_conf_noalloc: T=%d, V=%d exceed the fixed scratch (at most %d rows and a "
            "vocabulary of %d)\n",
            T, V, kNoAllocMaxRows, kNoAllocMaxTiles * 256);
    return DLLM_E_INVAL;
  }
  dllm_handle tmp;
  tmp.st = reinterpret_cast<cudaStream_t>(stream);
  dllm_handle* h = &tmp;
  unsigned char* base = nullptr;
  CK(noalloc_scratch(&base));
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, y, T, d, 128) || !make_tmap(&tb, head, V, d, 256)) return DLLM_E_INVAL;
  const int nvt = V / 256;
  float* pm = reinterpret_cast<float*>(base);
  float* ps = pm + kNoAllocPartials;
  int32_t* pi = reinterpret_cast<int32_t*>(ps + kNoAllocPartials);
  int* err = reinterpret_cast<int*>(pi + kNoAllocPartials);
  // the partials are fully rewritten for rows < T; only the error word must start at zero
  CK(cudaMemsetAsync(err, 0, sizeof(int), tmp.st));
  tmp.d_err = err;
  const int mt = ceil_div(T, 128);
  DenseSched s{T, mt, 256};
  EpiLMHead<256> e{pm, ps, pi, nvt, mask_id};
  cudaError_t r = launch_gemm<256, 4, 1, kSplitNone>(h, dim3(mt * nvt), ta, tb, d / 64, 0, s, e);
  if (r == cudaSuccess) {
    lm_merge_kernel<<<ceil_div((long)T * 32, 256), 256, 0, tmp.st>>>(pm, ps, pi, T, nvt, conf, argmax, err);
    r = cudaGetLastError();
  }
  tmp.d_err = nullptr;
  return r == cudaSuccess ? DLLM_OK : DLLM_E_CUDA;
}
