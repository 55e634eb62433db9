/*
 * dllm.h - C ABI of the B200 masked block-diffusion denoiser (libdllm.so).
 *
 * The calls follow the problem as the pages state it ("Diffusion LLMs: what changes
 * when you stop generating one token at a time", below "What changes"; "Diffusion
 * LLMs are not a good fit for distributed inference", below "Distributed"):
 *   - dllm_prefill: causal prefill of the prompt into the KV cache
 *     (What changes, section 4.2, "Block decoding": prefill is causal);
 *   - dllm_denoise_step: one forward pass over a 256-position canvas with
 *     bidirectional attention to the cached prefix and to the canvas itself, the
 *     per-position confidence (max softmax probability) and argmax, and a commit of the
 *     most confident still-[MASK] positions (What changes, section 2, "Reverse
 *     (generation) process" and its two properties; section 5, "Quality vs steps",
 *     for the confidence threshold);
 *   - dllm_generate_block: denoising steps until the canvas is full or the step budget
 *     is spent (What changes, section 4.2, "Few steps": up to 48 steps; Distributed,
 *     the canvas paragraph);
 *   - dllm_append_kv: the finished canvas joins the KV cache (What changes, section 4.2,
 *     "Block decoding"; section 4.1, block diffusion: autoregressive across blocks);
 *   - dllm_generate: the end-to-end request (prompt in, canvases out) with host buffers.
 *
 * Conventions
 *   - Every call returns DLLM_OK (0) or a negative DLLM_E_* code; no C++ exception
 *     crosses the ABI. dllm_last_error() returns the handle's last message.
 *   - "device" pointers are CUDA device memory owned by the caller; "host" pointers are
 *     ordinary host memory owned by the caller. The handle owns its repacked weights, the
 *     KV cache, all scratch and its CUDA graphs.
 *   - All GPU work is ordered on the stream given to dllm_create. Calls return once the
 *     work is queued, except dllm_create, dllm_generate_block, dllm_generate, dllm_check,
 *     dllm_set_debug / dllm_debug_* and dllm_set_wait_limit, which synchronise that
 *     stream. dllm_prefill and dllm_generate with a host prompt copy it before returning.
 *   - Device-side errors: every wait inside a kernel is bounded. A kernel that gives up
 *     one records an error word on the device and returns; the context stays usable.
 *     The pass that saw it commits nothing (remaining = -1, conf = NaN, argmax = -1),
 *     later passes commit nothing either, and the next synchronising call (dllm_check,
 *     dllm_generate_block, dllm_generate) returns DLLM_E_TIMEOUT and clears the word.
 *   - Canvas layout: int32 tokens [B][C] and uint8 mask [B][C] (1 = still [MASK]); request
 *     b of a batched call uses KV slot b. Masked positions hold mask_id.
 *   - Not thread-safe: one host thread per handle.
 */
#ifndef DLLM_H_
#define DLLM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DLLM_OK 0
#define DLLM_E_INVAL (-1)     /* bad argument or unsupported shape */
#define DLLM_E_OOM (-2)       /* device allocation failed */
#define DLLM_E_CUDA (-3)      /* CUDA runtime / driver error */
#define DLLM_E_CTX_FULL (-4)  /* the KV cache cannot hold the prefix plus a canvas */
#define DLLM_E_BUDGET (-5)    /* step budget spent with positions still masked */
#define DLLM_E_STATE (-6)     /* call out of order (e.g. a canvas pass before prefill) */
#define DLLM_E_TIMEOUT (-7)   /* a kernel gave up a bounded wait; the context is intact */

#define DLLM_WEIGHTS_F32 0
#define DLLM_WEIGHTS_BF16 1

#define DLLM_EXPERTS_BF16 0
#define DLLM_EXPERTS_FP8 1

#define DLLM_POLICY_TOPK 0
#define DLLM_POLICY_THRESHOLD 1

typedef struct dllm_handle dllm_handle;

/* Model and capacity. Requirements of this library: d_model % 256 == 0, d_model <= 4096,
 * head_dim in {64, 176}, n_heads * head_dim % 64 == 0, ffn_dim % 64 == 0,
 * vocab % 256 == 0, n_experts <= 256, top_k <= 8 (dense: n_experts = 0, top_k = 1),
 * canvas <= 1024, mask_id = vocab - 1. */
typedef struct {
  int n_layers, d_model, n_heads, n_kv_heads, head_dim;
  int n_experts;   /* 0 = dense SwiGLU FFN */
  int top_k, ffn_dim, vocab, mask_id, canvas;
  int max_ctx;     /* KV positions per request; a canvas pass needs prefix + canvas <= max_ctx */
  int max_batch;   /* requests (KV slots) */
  float rms_eps;   /* 1e-6 */
  float rope_theta;/* 10000 */
  int weight_dtype;/* DLLM_WEIGHTS_F32 or DLLM_WEIGHTS_BF16 */
  /* DLLM_EXPERTS_BF16 (0): expert weights as given. DLLM_EXPERTS_FP8 (1): at create, every
   * expert matrix (Wg, Wu, Wd) is stored as FP8 E4M3 with one power-of-two scale 2^e per
   * 128 x 128 tile of the matrix, e the least integer with the tile's max |w| <= 448 * 2^e,
   * codes rounded to nearest even (What changes, section 4.2 "Speed": the measured setting
   * runs FP8). The kernels expand each staged tile to bf16 exactly, so the pass computes on
   * the FP8 values; expert bytes per pass halve. */
  int expert_format;
} dllm_config;

/* Commit policy (What changes, section 2 and section 5).
 * TOPK: commit the min(k, R) most confident masked positions.
 * THRESHOLD: commit every masked position with conf > tau; with floor = 1 commit at
 * least max(1, ceil(R / (max_steps - step))) of the most confident ones, so that the
 * canvas completes within max_steps. Ties go to the lower position.
 * t2t = 1 adds token-to-token editing (What changes, section 4.3, LLaDA2.1's T2T next
 * to mask-to-token decoding): a position committed before the pass is re-written to the
 * pass's argmax when that token differs from its own and conf > edit_tau; it stays
 * committed, and R counts masked positions only. t2t = 0 (a zeroed struct): committed
 * tokens never change. */
typedef struct {
  int kind;
  int k;
  float tau;
  int floor;
  int t2t;
  float edit_tau;
} dllm_policy;

/* Creates a handle. `weights` is the blob in this order, every tensor row-major
 * [out][in] in weight_dtype, each starting on a 256-byte boundary:
 *   emb[V][d]; per layer: attn_norm[d], Wq[H*hd][d], Wk[Hkv*hd][d], Wv[Hkv*hd][d],
 *   Wo[d][H*hd], ffn_norm[d], then Wr[E][d] and per expert Wg[F][d], Wu[F][d], Wd[d][F]
 *   (dense: Wg, Wu, Wd); final_norm[d]; head[V][d].
 * weights_on_device: 1 if `weights` is device memory, 0 for host memory. The blob is
 * copied and repacked; the caller may free it after the call returns.
 * cuda_stream: a cudaStream_t, used as given; NULL: the handle creates its own non-blocking
 *   stream (destroyed with the handle).
 * Errors: DLLM_E_INVAL (shape), DLLM_E_OOM, DLLM_E_CUDA. On error *out is NULL. */
int dllm_create(const dllm_config* cfg, const void* weights, size_t weight_bytes, int weights_on_device,
                void* cuda_stream, dllm_handle** out);

/* Causal prefill of request slot `req`: prompt (device int32 [n]) at positions 0..n-1;
 * replaces that slot's cache. Errors: DLLM_E_INVAL, DLLM_E_CTX_FULL (n + canvas > max_ctx). */
int dllm_prefill(dllm_handle* h, int req, const int32_t* prompt, int n);

/* One denoising pass over requests 0..req_count-1 followed by a commit.
 * canvas (device int32 [req_count][C]) and mask (device uint8 [req_count][C]) are read
 * and updated in place. step is the 0-based step index (used by the threshold floor).
 * conf_out (device float [req_count][C]) and argmax_out (device int32 [req_count][C])
 * receive the pass's confidence and argmax of every position when not NULL.
 * remaining_out (device int32 [req_count]) receives the masked count after the commit.
 * Returns once the pass is queued; it reads no device result, so a kernel that gave
 * up a bounded wait shows as remaining_out = -1, conf_out = NaN and argmax_out = -1 of
 * that pass (nothing committed), and as DLLM_E_TIMEOUT from the next dllm_check.
 * Errors: DLLM_E_INVAL, DLLM_E_STATE (slot without prefill), DLLM_E_CTX_FULL. */
int dllm_denoise_step(dllm_handle* h, int req_count, int32_t* canvas, uint8_t* mask, const dllm_policy* policy,
                      int step, int max_steps, float* conf_out, int32_t* argmax_out, int32_t* remaining_out);

/* Denoises fresh all-[MASK] canvases of requests 0..req_count-1 until every position is
 * committed or max_steps passes ran. canvas_out: device int32 [req_count][C] or NULL.
 * steps_taken: host int [req_count] or NULL. Synchronises the stream.
 * Errors: as dllm_denoise_step, DLLM_E_BUDGET (positions left after max_steps),
 * DLLM_E_TIMEOUT. */
int dllm_generate_block(dllm_handle* h, int req_count, int max_steps, const dllm_policy* policy,
                        int32_t* canvas_out, int* steps_taken);

/* Appends finished canvases (device int32 [req_count][C]; NULL = the handle's last
 * generated canvases) to the KV cache: one bidirectional pass whose K/V are kept at
 * positions P..P+C-1; each request's prefix then grows by C. */
int dllm_append_kv(dllm_handle* h, int req_count, const int32_t* canvas);

/* Approximate append (What changes, section 5, "KV caching": Fast-dLLM's training-free,
 * block-wise approximate KV cache): the K/V that each request's last canvas pass wrote
 * at positions P..P+C-1 are kept as the finished canvas's cache entries, with no extra
 * pass; each prefix grows by C. Those K/V were computed while the positions that pass
 * committed were still [MASK], so later passes see a slightly different cache than after
 * dllm_append_kv. Errors: DLLM_E_STATE (a slot without a canvas pass since its last
 * prefill or append), DLLM_E_CTX_FULL, DLLM_E_INVAL. */
int dllm_append_kv_approx(dllm_handle* h, int req_count);

/* End to end with host buffers: for each request r < req_count, prefill
 * prompts[r][0..n_prompt-1], then n_canvases times generate a canvas and append it.
 * tokens_out: host int32 [req_count][n_canvases * C]; steps_out: host int
 * [req_count * n_canvases] or NULL (steps per canvas, the maximum over requests is
 * what the batch ran). Synchronises the stream. */
int dllm_generate(dllm_handle* h, int req_count, const int32_t* prompts, int n_prompt, int n_canvases,
                  int max_steps, const dllm_policy* policy, int32_t* tokens_out, int* steps_out);

/* Drops request slot req's KV cache (prefix length 0). */
int dllm_reset(dllm_handle* h, int req);

/* Prefix length of slot req, or a negative code. */
int dllm_prefix_len(const dllm_handle* h, int req);

/* Synchronises the stream and reports a device-side error (DLLM_E_TIMEOUT) or a CUDA
 * error raised since the last check. */
int dllm_check(dllm_handle* h);

/* Kernel launches issued by the handle since creation (graph replays count their
 * kernels). */
long long dllm_launch_count(const dllm_handle* h);

/* Limit, in nanoseconds, of the pipeline waits inside the kernels (a stage waiting for
 * its TMA copy, an MMA for its operands, an epilogue for its accumulator, a split-K
 * rank for its peers); ns <= 0 restores the default of 2 s. A wait first suspends for up
 * to 256 ns and counts the limit from there, so a wait that completes within that
 * window never gives up, whatever the limit. The waits that let copies
 * and MMAs already in flight land before a kernel exits keep the default. The limit is
 * one value per device, shared by every handle on it; it exists so that the timeout
 * path (DLLM_E_TIMEOUT, context intact) can be exercised. Synchronises the stream. */
int dllm_set_wait_limit(dllm_handle* h, long long ns);

/* Debug inspection of the last canvas pass (enable first; enabling drops captured
 * graphs). what: 0 = final residual x, fp32 [T][d]; 1 = router logits of `layer`,
 * fp32 [T][E]; 2 = top-k experts of `layer`, int32 [T][k]; 3 = conf, fp32 [T];
 * 4 = argmax, int32 [T]; 5 = residual after `layer`, fp32 [T][d]; 6 / 7 = K / V cache
 * of `layer` for slot 0, bf16 [Hkv][max_ctx][hd]. dst is host memory of `bytes` bytes,
 * T = req_count * C of the last pass. Synchronises the stream. */
int dllm_set_debug(dllm_handle* h, int on);
int dllm_debug_read(dllm_handle* h, int what, int layer, void* dst, size_t bytes);

/* Debug (needs dllm_set_debug(h, 1)): later passes over T tokens (canvas passes,
 * prefill or append, whichever has exactly T tokens) use the given experts instead of
 * their own top-k, layer by layer (idx: host int32 [n_layers][T][k]);
 * gates come from the pass's own router logits at those experts. The router's own
 * choice is still recorded for dllm_debug_read(what = 2). This isolates one layer's
 * routing decision from near-tie flips in earlier layers when comparing with a
 * reference. idx = NULL switches it off. Errors: DLLM_E_STATE (debug off),
 * DLLM_E_INVAL (dense model, T or an index out of range). */
int dllm_debug_force_routing(dllm_handle* h, const int32_t* idx, int T);

/* Kernel timing: dllm_set_timing(h, kinds) with kinds a bit mask of (1 << DLLM_TIMING_*)
 * (0 = off). Every later canvas pass then brackets the chosen kernel groups of each
 * layer with CUDA events (recorded inside the pass's CUDA graph); the elapsed times
 * are summed per kind after each pass of dllm_generate_block. dllm_timing_read fills
 * total_ms[kind], launches[kind] and bytes[kind] (arrays of DLLM_TIMING_KINDS); bytes
 * are filled for the two grouped GEMMs: the launches' algorithmic HBM bytes, i.e. the
 * bf16 weights of the experts each layer routed to plus the token rows read and the
 * results written, both counted at bf16 size (2 bytes per element). If reset, the sums
 * are zeroed. Changing the mask drops captured
 * graphs. Kinds: grouped gate/up GEMM; grouped down GEMM; attention (+ split merge);
 * QKV GEMM; O GEMM; routing (pre-FFN RMSNorm, router, top-k, permute, gather);
 * combine of the expert outputs (with the next RMSNorm fused into it);
 * LM head (final RMSNorm, LM-head GEMM, merge, commit; one per pass).
 * Bits 16..23 of kinds, if nonzero, give a layer stride S: only layers l % S == 0 are
 * bracketed (fewer event nodes in the graph, so the timed pass runs closer to an
 * untimed one); launches[] counts the bracketed launches only. */
#define DLLM_TIMING_STRIDE_SHIFT 16
#define DLLM_TIMING_GATE_UP 0
#define DLLM_TIMING_DOWN 1
#define DLLM_TIMING_ATTN 2
#define DLLM_TIMING_QKV 3
#define DLLM_TIMING_OPROJ 4
#define DLLM_TIMING_ROUTE 5
#define DLLM_TIMING_NORM 6
#define DLLM_TIMING_HEAD 7
#define DLLM_TIMING_KINDS 8
int dllm_set_timing(dllm_handle* h, int kinds);
int dllm_timing_read(dllm_handle* h, double* total_ms, long long* launches, double* bytes, int reset);

const char* dllm_last_error(const dllm_handle* h);
void dllm_destroy(dllm_handle* h);

/* ---- single-operation entry points (the pass's kernels on caller buffers) ---------
 * All pointers are device memory, stream = cudaStream_t. They validate shapes, queue
 * the work and return; errors as above. They return before the kernels run, so a
 * kernel that gives up a bounded wait is reported in the outputs instead: the GEMM
 * fills D with NaN, the LM heads write conf = NaN and argmax = -1 in every row. */

/* D[M][N] (fp32, row-major) = A[M][K] * B[N][K]^T with bf16 A, B; the tcgen05 GEMM core.
 * K % 64 == 0, N % 128 == 0. */
int dllm_op_gemm_bf16(const uint16_t* A, const uint16_t* B, float* D, int M, int N, int K, void* stream);

/* The FP8 block quantiser that dllm_create applies to expert matrices with
 * DLLM_EXPERTS_FP8: w (bf16 [rows][cols], row-major) -> q (E4M3 codes [rows][cols]) and
 * exps (int8 [ceil(rows/128)][ceil(cols/128)]): per 128 x 128 tile, e = the least integer
 * with max |w| <= 448 * 2^e (0 for an all-zero tile), q = nearest E4M3 (ties to even) of
 * w * 2^-e. cols % 16 == 0. */
int dllm_op_quantize_fp8(const uint16_t* w, int rows, int cols, uint8_t* q, int8_t* exps, void* stream);

/* The fused LM head (What changes, section 2: commit the most confident positions):
 * for each of the T rows of y (bf16 [T][d]) against head (bf16 [V][d]), argmax over
 * the vocabulary without mask_id (ties to the lowest id) and conf = 1 / sum_v exp(l_v -
 * max). conf: float [T]; argmax: int32 [T]. Needs d % 64 == 0, V % 256 == 0. Allocates
 * and frees its own partial-result scratch (stream-ordered). */
int dllm_op_lm_head_conf(const uint16_t* y, const uint16_t* head, int T, int d, int V, int mask_id, float* conf,
                         int32_t* argmax, void* stream);

/* dllm_op_lm_head_conf without any device allocation. The pages have no counterpart:
 * this entry point exists for callers that cannot allocate device memory while they
 * run, e.g. a host process that reserves the whole device for its own allocator under
 * a fixed budget and forbids other cudaMalloc calls, or a path where an allocation's
 * implicit synchronisation or failure is not acceptable.
 * Arguments and results are those of dllm_op_lm_head_conf (caller-owned device buffers).
 * Scratch: one fixed device array inside the library (3 MiB). The CUDA runtime reserves
 * it on a device when it loads the library's module there, which it may do lazily, at
 * the library's first call on that device (whichever entry point that is); from then on
 * the device holds it until the process exits. A caller with a fixed device budget
 * should therefore make one call into the library on each device before its own
 * allocator takes the device. Limits: T <= 1024 rows, V <= 65536; larger sizes return
 * DLLM_E_INVAL and print the limit to stderr.
 * The first call on a device looks up that array's device address (once per device,
 * with the device current) and keeps it; make that first call before any stream
 * capture, and do not keep calling across a cudaDeviceReset of that device (the array
 * may move when the module is loaded again).
 * Every call on a device shares the one array and it keeps the last call's contents:
 * calls that may overlap on the GPU (other streams, other host threads) race on it, so
 * order them on one stream. Calls no cudaMalloc, cudaFree or allocating library
 * routine. */
int dllm_op_lm_head_conf_noalloc(const uint16_t* y, const uint16_t* head, int T, int d, int V, int mask_id,
                                 float* conf, int32_t* argmax, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DLLM_H_ */
