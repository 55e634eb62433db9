// Tensor-core GEMM for sm_100a: D[128 x BN] = A[128 x K] * B[BN x K]^T per tile, bf16
// operands staged by TMA into 128-byte-swizzled shared memory, tcgen05.mma issued by one
// thread, fp32 accumulators in TMEM, and a fused epilogue that reads TMEM row by row.
//
// Roles (192 threads): warp 0 lane 0 issues TMA loads; warp 1 owns the TMEM allocation
// and lane 0 issues the MMAs; warps 2..5 run the epilogue, warp w reading TMEM lanes
// 32*(w%4)..32*(w%4)+31 (one accumulator row per thread). Stages are handed over with
// mbarriers (full: TMA bytes landed; empty: the MMAs reading the stage completed), the
// accumulator with acc_full / acc_empty so that, when a CTA owns several tiles, the
// epilogue of one overlaps the main loop of the next. Every wait is bounded.
#pragma once

#include "common.cuh"

namespace dllm {

struct Tile {
  int a_row;     // A tensor-map row of the tile's first row
  int b_row;     // B tensor-map row of the tile's first column
  int m_valid;   // rows of the tile inside the problem
  int n_valid;   // columns of the tile inside the problem
  int mt, nt;    // dense: (m tile, n tile); grouped: (m tile inside the expert, expert)
  int m_count = 1;   // m tiles of this work item (128 rows apart, sharing the B tile)
  int n_cols = 0;    // accumulator columns computed (per operand half); 0 = the full BN
  int ks = 0;        // K slice of a DensePartKSched tile (its epilogue writes partial ks)
};

// Columns of the tile an epilogue reads: the full BN, or the rounded-up valid columns
// of a grouped tile whose MMA width follows its token count.
template <int BN>
DLLM_DEV int tile_cols(const Tile& t) { return t.n_cols > 0 ? t.n_cols : BN; }

// One output tile per CTA over an M x N problem; m tiles vary fastest so that the CTAs
// sharing a weight tile run close together (the second read hits L2).
struct DenseSched {
  static constexpr int kSmemBytes = 0;
  static constexpr int kKSplit = 1;
  static constexpr bool kPartK = false;
  static constexpr bool kDynN = false;
  static constexpr bool kW8 = false;
  static constexpr int kMPerItem = 1;
  int M, n_mtiles, BN;
  DLLM_DEV void stage(int*) {}
  DLLM_DEV int count() const { return 1; }
  DLLM_DEV Tile tile(int) const {
    Tile t;
    int id = blockIdx.x;
    t.mt = id % n_mtiles;
    t.nt = id / n_mtiles;
    t.a_row = t.mt * 128;
    t.b_row = t.nt * BN;
    t.m_valid = min(128, M - t.a_row);
    t.n_valid = BN;
    return t;
  }
};

// Dense tiles with the K loop split over a cluster of KS CTAs (consecutive blockIdx.x):
// CTA rank r of a cluster accumulates k blocks [r*kb/KS, (r+1)*kb/KS) of the same output
// tile, and the partial sums meet in rank 0's TMEM over distributed shared memory
// before the epilogue. For problems with fewer tiles than SMs.
template <int KS>
struct DenseSplitKSched {
  static constexpr int kSmemBytes = 0;
  static constexpr int kKSplit = KS;
  static constexpr bool kPartK = false;
  static constexpr bool kDynN = false;
  static constexpr bool kW8 = false;
  static constexpr int kMPerItem = 1;
  int M, n_mtiles, BN;
  DLLM_DEV void stage(int*) {}
  DLLM_DEV int count() const { return 1; }
  DLLM_DEV Tile tile(int) const {
    Tile t;
    int id = blockIdx.x / KS;
    t.mt = id % n_mtiles;
    t.nt = id / n_mtiles;
    t.a_row = t.mt * 128;
    t.b_row = t.nt * BN;
    t.m_valid = min(128, M - t.a_row);
    t.n_valid = BN;
    return t;
  }
};

// Dense tiles with the K loop split over `ks` independent CTAs (consecutive blockIdx.x,
// no cluster): slice r accumulates k blocks [r*kb/ks, (r+1)*kb/ks) and its epilogue
// writes partial sum r of the tile (Tile::ks) to global memory, where the consumer kernel
// adds the ks partials in slice order. No CTA waits on another, so the slices need not be
// co-resident and nothing stalls at the end of the K loop.
struct DensePartKSched {
  static constexpr int kSmemBytes = 0;
  static constexpr int kKSplit = 1;
  static constexpr bool kPartK = true;
  static constexpr bool kDynN = false;
  static constexpr bool kW8 = false;
  static constexpr int kMPerItem = 1;
  int M, n_mtiles, BN, ks;
  DLLM_DEV void stage(int*) {}
  DLLM_DEV int count() const { return 1; }
  DLLM_DEV Tile tile(int) const {
    Tile t;
    int id = blockIdx.x / ks;
    t.ks = blockIdx.x % ks;
    t.mt = id % n_mtiles;
    t.nt = id / n_mtiles;
    t.a_row = t.mt * 128;
    t.b_row = t.nt * BN;
    t.m_valid = min(128, M - t.a_row);
    t.n_valid = BN;
    return t;
  }
};

// Persistent grouped schedule over the routed experts only. One work item is MPI output
// tiles that share their token chunk: (routed expert r, m tiles MPI*g .. MPI*g+MPI-1,
// token chunk of BN), so the chunk's B tile is loaded once for MPI weight tiles. Items
// of expert r are numbered g * chunks_r + chunk from m_groups * chunk_prefix[r] on, so
// the chunks of one weight tile are neighbours: CTAs running them together read that
// tile from HBM once and from L2 after. CTA c takes items c, c + gridDim.x, ...: every CTA gets the same
// number of equal-sized tiles whatever the routing skew, and streams them back to back
// (the next tile's loads overlap this tile's epilogue through the double-buffered
// accumulator).
//
// The routing tables are copied into shared memory once per CTA (stage(), run by every
// thread before the roles split), so that finding an item's expert is a short search in
// shared memory instead of a chain of dependent global loads on the producer's path.
//
// With DYN (kDynN) the MMA width follows each chunk's token count: a chunk of n tokens
// loads only n16 = n rounded up to 16 rows of the token pair (a full chunk with the
// BN-row boxes of tma_b / tma_b2, a partial one composed from the kernel's TokMaps boxes
// of 64, 32 and 16 rows), stacked as [hi n16 rows | lo n16 rows], and one MMA of N = 2 n16
// reads both. Without it every chunk loads and multiplies BN token rows (the rows past
// the chunk's end belong to the next expert and are dropped by the epilogue); measured
// faster at batch 1 both at random-init routing (gate/up 64 vs 80 us per 26B canvas
// launch) and with every expert routed (187 vs 229 us), so the engine runs the fixed
// width; the dynamic one stays available to the schedules.
//
// W8: the weights are FP8 E4M3 with one power-of-two scale 2^e per 128 x 128 tile of
// each original expert matrix (exps, int8). Converter warps turn each staged FP8 tile
// into bf16 (exact) straight into tensor memory, where the MMA reads its A operand, so
// the bf16 copy never touches shared memory. exp_interleave = 1 for the gate/up layout
// (each 128-row tile: 64 gate rows, then the matching 64 up rows), 0 for down; exps is
// [E][2 if interleaved][exp_nrb][exp_ncb].
template <int MPI, bool W8 = false, bool DYN = false>
struct PersistentGroupedSched {
  static constexpr int kMaxRouted = 256;
  static constexpr int kSmemBytes = (4 * kMaxRouted + 8) * 4;
  static constexpr int kKSplit = 1;
  static constexpr bool kPartK = false;
  static constexpr bool kDynN = DYN;
  static constexpr bool kW8 = W8;
  static constexpr int kMPerItem = MPI;
  const int* offsets;        // [E+1] token ranges per expert
  const int* routed;         // [E] experts with at least one token, ascending
  const int* n_routed;       // [1]
  const int* chunk_prefix;   // [n_routed + 1] prefix sums of ceil(count / BN) over routed
  int rows_per_expert;
  int m_tiles;
  int BN;
  const int8_t* exps = nullptr;
  int exp_interleave = 0, exp_nrb = 0, exp_ncb = 0;
  // scale exponent of row r of m tile u of tile t at k block kb (64 columns)
  DLLM_DEV int exponent(const Tile& t, int u, int r, int kb) const {
    const int mt = t.mt + u;
    const int cb = kb >> 1;
    if (exp_interleave) return exps[((t.nt * 2 + (r >> 6)) * exp_nrb + (mt >> 1)) * exp_ncb + cb];
    return exps[(t.nt * exp_nrb + mt) * exp_ncb + cb];
  }
  // shared-memory copies, per routed expert r: token offset and count (set by stage())
  const int* s_off = nullptr;
  const int* s_cnt = nullptr;
  DLLM_DEV void stage(int* s) {
    const int n = min(*n_routed, kMaxRouted);
    int* cp = s;
    int* ex = cp + kMaxRouted + 1;
    int* of = ex + kMaxRouted;
    int* ct = of + kMaxRouted;
    int* nn = ct + kMaxRouted;
    for (int i = threadIdx.x; i <= n; i += blockDim.x) {
      cp[i] = chunk_prefix[i];
      if (i < n) {
        const int e = routed[i];
        const int o = offsets[e];
        ex[i] = e;
        of[i] = o;
        ct[i] = offsets[e + 1] - o;
      }
    }
    if (threadIdx.x == 0) *nn = n;
    chunk_prefix = cp;
    routed = ex;
    s_off = of;
    s_cnt = ct;
    n_routed = nn;
  }
  DLLM_DEV int m_groups() const { return (m_tiles + MPI - 1) / MPI; }
  DLLM_DEV int n_items() const { return chunk_prefix[*n_routed] * m_groups(); }
  DLLM_DEV int count() const {
    const int n = n_items();
    return (int)blockIdx.x < n ? (n - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  }
  DLLM_DEV Tile tile(int j) const {
    const int i = blockIdx.x + j * gridDim.x;
    const int mg = m_groups();
    int lo = 0, hi = *n_routed;   // chunk_prefix[lo] * mg <= i < chunk_prefix[hi] * mg
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (chunk_prefix[mid] * mg <= i) lo = mid; else hi = mid;
    }
    const int e = routed[lo];
    const int ch = chunk_prefix[lo + 1] - chunk_prefix[lo];
    const int local = i - chunk_prefix[lo] * mg;
    const int chunk = local % ch;
    const int off = s_off[lo];
    const int cnt = s_cnt[lo];
    Tile t;
    t.mt = (local / ch) * MPI;
    t.m_count = min(MPI, m_tiles - t.mt);
    t.nt = e;
    t.a_row = e * rows_per_expert + t.mt * 128;
    t.b_row = off + chunk * BN;
    t.m_valid = 128;
    t.n_valid = min(BN, cnt - chunk * BN);
    t.n_cols = kDynN ? (t.n_valid + 15) & ~15 : 0;
    return t;
  }
};

// The token-operand tensor maps of a dynamic-width grouped GEMM, passed by value as a
// kernel parameter: [hi boxes of 16, 32, 64, 128 rows | lo boxes of the same heights].
struct alignas(64) TokMaps {
  CUtensorMap m[8];
};

__host__ __device__ constexpr int tmem_cols_for(int bn) {
  return bn <= 32 ? 32 : bn <= 64 ? 64 : bn <= 128 ? 128 : 256;
}

// tcgen05.alloc takes a power of two of at least 32 columns.
__host__ __device__ constexpr int tmem_alloc_cols(int n) {
  return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512;
}

// Threads of a GEMM CTA: producer, MMA, 4 epilogue warps, and for W8 8 converter warps
// (two per TMEM lane quarter, each on half of a row's 64 k values).
template <class Sched>
__host__ __device__ constexpr int gemm_threads() { return Sched::kW8 ? 448 : 192; }
constexpr int kConvThreads = 256;
constexpr int kConvMaxColBlocks = 64;   // W8: 128-column scale blocks per weight row (K <= 8192)

// Operand splitting. Weights are bf16; an activation operand can be carried as a pair
// of bf16 tensors (hi = bf16(v), lo = bf16(v - hi)) so that products keep about 16
// mantissa bits of the activation. kSplitNone: plain. kSplitA: A is a (hi, lo) pair and
// every k step issues two MMAs into the same accumulator. kSplitB: B is the pair; its
// hi and lo rows sit next to each other in the stage, one MMA of width 2 BN reads both,
// and the epilogue first adds the accumulator's two column halves. kSplitA3: A is a
// triple (hi, mid, lo) carrying all 24 bits of an fp32 value, three MMAs per k step (the
// third map travels in the TokMaps parameter's first slot).
enum SplitMode : int { kSplitNone = 0, kSplitA = 1, kSplitB = 2, kSplitA3 = 3 };

template <int BN, int STAGES, int SPLIT, class Epi, class Sched = DenseSched>
struct GemmSmem {
  // one 128-row A tile of a k block: bf16, or FP8 bytes for a W8 schedule
  static constexpr int kAtile = Sched::kW8 ? 128 * 64 : 128 * 64 * 2;
  static constexpr int kA = Sched::kMPerItem * kAtile;     // the item's A tiles
  static constexpr int kB = BN * 64 * 2;
  static constexpr int kA2 = (SPLIT == kSplitA || SPLIT == kSplitA3) ? kA : 0;
  static constexpr int kA3 = SPLIT == kSplitA3 ? kA : 0;
  static constexpr int kB2 = SPLIT == kSplitB ? kB : 0;
  static constexpr int kStageBytes = kA + kA2 + kA3 + kB + kB2;   // TMA bytes per stage
  static constexpr int kOffA2 = STAGES * kA;
  static constexpr int kOffA3 = kOffA2 + STAGES * kA2;
  static constexpr int kOffB = kOffA3 + STAGES * kA3;
  // kSplitB keeps each stage's B pair adjacent ([hi rows | lo rows]), so that one MMA
  // with N = 2 BN reads both: the A tile is then read from shared memory once per k step
  // instead of once per half.
  static constexpr int kBStage = kB + kB2;
  static constexpr int kOffB2 = kOffB + kB;   // the lo half of stage 0 (stage s: + s * kBStage)
  // W8: the converted bf16 A tiles, one per stage, 128-byte swizzled like a TMA-loaded tile
  static constexpr int kAbf = Sched::kW8 ? Sched::kMPerItem * 128 * 64 * 2 : 0;
  static constexpr int kOffAbf = STAGES * kStageBytes;
  static constexpr int kBarOff = kOffAbf + STAGES * kAbf;
  static constexpr int kEpiOff = kBarOff + 256;
  static constexpr int kSchedOff = kEpiOff + Epi::kSmemBytes;
  static constexpr int kTotal = kSchedOff + Sched::kSmemBytes + 1024;   // + alignment slack
};

DLLM_DEV void epi_bar_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// True on every epilogue thread iff it is true on all 128 of them (named barrier 1).
DLLM_DEV bool epi_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)ok)
      : "memory");
  return r != 0;
}

// Split-K hand-over of one tile's partial sums inside a cluster (epilogue threads only;
// thread r owns accumulator row r). Ranks > 0 copy their TMEM partial into their own
// shared memory ([BN/4][128] float4, over the stage buffers, idle once the tile's last
// MMA has completed) and signal rank 0, which adds every peer's partial into its TMEM
// accumulator through distributed shared memory. The cluster barrier at the end of the
// kernel keeps the peers resident until rank 0 has read them. Returns false (with *err
// set) when the wait runs out.
template <int BN, int KS>
DLLM_DEV bool splitk_reduce(int krank, uint32_t taddr, int r, uint8_t* part_smem, uint64_t* peer_ready,
                            volatile int* abort_flag, int* err) {
  float4* part = reinterpret_cast<float4*>(part_smem);
  if (krank != 0) {
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      tmem_ld16(taddr + c, v);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        part[((c >> 2) + i) * 128 + r] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
    mbar_arrive_cluster(mapa_shared(smem_u32(peer_ready), 0));
    return true;
  }
  const bool got = mbar_wait_cluster(peer_ready, 0, abort_flag);
  if (!epi_all(got)) {
    if (!got) atomicExch(err, kDevTimeoutEpilogue);
    return false;
  }
#pragma unroll 1
  for (int p = 1; p < KS; ++p) {
    const uint32_t base = mapa_shared(smem_u32(part), p);
    // up to 64 columns at a time: the remote loads are issued together, then added
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 64) {
      float4 w[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (c0 + 4 * i < BN) w[i] = ld_shared_cluster_v4(base + (uint32_t)((((c0 >> 2) + i) * 128 + r) * 16));
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c = c0 + 16 * q;
        if (c >= BN) break;   // uniform
        float v[16];
        tmem_ld16(taddr + c, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[4 * i] += w[4 * q + i].x;
          v[4 * i + 1] += w[4 * q + i].y;
          v[4 * i + 2] += w[4 * q + i].z;
          v[4 * i + 3] += w[4 * q + i].w;
        }
        tmem_st16(taddr + c, v);
      }
    }
  }
  return true;
}

template <int BN, int STAGES, int ACC_BUFS, int SPLIT, class Sched, class Epi>
__global__ void __launch_bounds__(gemm_threads<Sched>(), 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_a2,
               const __grid_constant__ CUtensorMap tma_b, const __grid_constant__ CUtensorMap tma_b2,
               const __grid_constant__ TokMaps tok, int k_blocks, int a_stream_first, Sched sched_in, Epi epi,
               int* err) {
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128 is a multiple of 16 in [16, 256]");
  using L = GemmSmem<BN, STAGES, SPLIT, Epi, Sched>;
  constexpr int kAccN = SPLIT == kSplitB ? 2 * BN : BN;   // kSplitB: columns [0, BN) hi, [BN, 2 BN) lo
  static_assert(kAccN <= 256, "UMMA N");
  constexpr int MPI = Sched::kMPerItem;                   // accumulators per work item
  static_assert(MPI == 1 || (SPLIT != kSplitA && SPLIT != kSplitA3), "several m tiles per item share B only");
  constexpr int kCols = tmem_cols_for(kAccN);
  constexpr bool W8 = Sched::kW8;
  static_assert(!W8 || SPLIT == kSplitB, "FP8 weights: grouped expert tiles only");
  constexpr int kAccCols = kCols * ACC_BUFS * MPI;
  constexpr int kTmemCols = tmem_alloc_cols(kAccCols);
  static_assert(kAccCols <= 512, "TMEM has 512 columns");
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, kAccN);
  constexpr int KS = Sched::kKSplit;
  static_assert(KS == 1 || BN * 128 * 4 <= STAGES * L::kStageBytes, "split-K partial fits the stage buffers");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sA2 = smem + L::kOffA2;
  uint8_t* sA3 = smem + L::kOffA3;
  uint8_t* sB = smem + L::kOffB;
  uint8_t* sB2 = smem + L::kOffB2;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + ACC_BUFS;
  uint64_t* drain = acc_empty + ACC_BUFS;
  uint64_t* peer_ready = drain + 1;   // split-K: rank 0 learns that the peers' partials are in place
  uint64_t* conv_full = drain + 2;    // W8: the stage's bf16 A tiles are in shared memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(conv_full + (W8 ? STAGES : 0));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* epi_smem = smem + L::kEpiOff;
  Sched sched = sched_in;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < ACC_BUFS; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    mbar_init(drain, 1);
    if (KS > 1) mbar_init(peer_ready, 128 * (KS - 1));
    if (W8)
      for (int s = 0; s < STAGES; ++s) mbar_init(&conv_full[s], kConvThreads);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tma_a);
    tma_prefetch_desc(&tma_b);
    if (SPLIT == kSplitA || SPLIT == kSplitA3) tma_prefetch_desc(&tma_a2);
    if (SPLIT == kSplitA3) tma_prefetch_desc(&tok.m[0]);
    if (SPLIT == kSplitB) tma_prefetch_desc(&tma_b2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (KS > 1) cluster_sync();   // the peers' barriers are initialised before anyone arrives on them
  pdl_trigger();                // after the TMEM allocation
  pdl_wait();                   // the inputs (and the routing tables) are complete from here on
  if (Sched::kSmemBytes > 0) {
    sched.stage(reinterpret_cast<int*>(smem + L::kSchedOff));
    __syncthreads();
  }
  const uint32_t tmem_base = *tmem_slot;
  const int ntiles = sched.count();
  const int krank = KS > 1 ? (int)cluster_ctarank() : 0;
  int kb_begin = krank * k_blocks / KS;
  int kb_end = (krank + 1) * k_blocks / KS;
  if constexpr (Sched::kPartK) {
    const int sl = (int)blockIdx.x % sched.ks;
    kb_begin = sl * k_blocks / sched.ks;
    kb_end = (sl + 1) * k_blocks / sched.ks;
  }

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    const uint64_t pol_first = policy_evict_first();
    const uint64_t pol_last = policy_evict_last();
    const uint64_t pol_a = a_stream_first ? pol_first : pol_last;
    const uint64_t pol_b = a_stream_first ? pol_last : pol_first;
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      const Tile t = sched.tile(j);
      for (int kb = kb_begin; kb < kb_end; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
        if constexpr (Sched::kDynN) {
          static_assert(SPLIT == kSplitB && BN <= 128 && BN % 16 == 0, "dynamic N: stacked token pair, <= 128 rows");
          const int n16 = t.n_cols;
          mbar_arrive_expect_tx(&full[stage], t.m_count * L::kAtile + 2 * n16 * 128);
          for (int u = 0; u < t.m_count; ++u)
            tma_load_2d(sA + stage * L::kA + u * L::kAtile, &tma_a, &full[stage], kb * 64, t.a_row + u * 128, pol_a);
          // [hi n16 rows | lo n16 rows]: a full chunk with the BN-row boxes of tma_b / tma_b2,
          // a partial one composed from boxes of 64 / 32 / 16 rows
          uint8_t* dst = sB + stage * L::kBStage;
          if (n16 == BN) {
            tma_load_2d(dst, &tma_b, &full[stage], kb * 64, t.b_row, pol_b);
            tma_load_2d(dst + BN * 128, &tma_b2, &full[stage], kb * 64, t.b_row, pol_b);
          } else {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              int off = 0;
#pragma unroll
              for (int bi = 2; bi >= 0; --bi) {
                const int rows = 16 << bi;
                if ((n16 - off) & rows) {
                  tma_load_2d(dst + (half * n16 + off) * 128, &tok.m[half * 4 + bi], &full[stage], kb * 64,
                              t.b_row + off, pol_b);
                  off += rows;
                }
              }
            }
          }
        } else {
          mbar_arrive_expect_tx(&full[stage], L::kStageBytes - (MPI - t.m_count) * L::kAtile);
          for (int u = 0; u < t.m_count; ++u)
            tma_load_2d(sA + stage * L::kA + u * L::kAtile, &tma_a, &full[stage], kb * 64, t.a_row + u * 128, pol_a);
          if (SPLIT == kSplitA || SPLIT == kSplitA3)
            tma_load_2d(sA2 + stage * L::kA2, &tma_a2, &full[stage], kb * 64, t.a_row, pol_a);
          if (SPLIT == kSplitA3) tma_load_2d(sA3 + stage * L::kA3, &tok.m[0], &full[stage], kb * 64, t.a_row, pol_a);
          tma_load_2d(sB + stage * L::kBStage, &tma_b, &full[stage], kb * 64, t.b_row, pol_b);
          if (SPLIT == kSplitB)
            tma_load_2d(sB2 + stage * L::kBStage, &tma_b2, &full[stage], kb * 64, t.b_row, pol_b);
        }
        ++issued;
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (!ok) {
      atomicExch(err, kDevTimeoutProducer);
      *abort_flag = 1;
      // let the copies already in flight land before the CTA's shared memory goes away
      int s = stage, p = phase;
      for (int i = 0; i < min(issued, STAGES); ++i) {
        s = (s + STAGES - 1) % STAGES;
        if (s == STAGES - 1) p ^= 1;
        mbar_drain(&full[s], p);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      const int acc = j % ACC_BUFS;
      const uint32_t acc_phase = (j / ACC_BUFS) & 1;
      if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      int mc = 1;
      uint32_t idesc = kIdesc;
      if constexpr (MPI > 1 || Sched::kDynN) {
        const Tile tj = sched.tile(j);
        mc = tj.m_count;
        if constexpr (Sched::kDynN) idesc = idesc_bf16_f32(128, 2 * tj.n_cols);
      }
      const uint32_t d_tmem = tmem_base + acc * MPI * kCols;
      for (int kb = kb_begin; kb < kb_end; ++kb) {
        if (!mbar_wait(W8 ? &conv_full[stage] : &full[stage], phase, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + stage * L::kA);
        const uint32_t b0 = smem_u32(sB + stage * L::kBStage);
        const uint32_t a1 = smem_u32(sA2 + stage * L::kA2);
        const uint32_t a2 = smem_u32(sA3 + stage * L::kA3);
        if constexpr (W8) {
          // A: the converted bf16 tile the converter warps wrote into shared memory
          const uint32_t ab = smem_u32(smem + L::kOffAbf + stage * L::kAbf);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int u = 0; u < MPI; ++u)
              if (u < mc)
                umma_bf16(d_tmem + u * kCols, sdesc_k_sw128(ab + u * 128 * 128 + kk * 32), sdesc_k_sw128(b0 + kk * 32),
                          idesc, (kb != kb_begin || kk != 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            umma_bf16(d_tmem, sdesc_k_sw128(a0 + kk * 32), sdesc_k_sw128(b0 + kk * 32), idesc,
                      (kb != kb_begin || kk != 0) ? 1u : 0u);
            if (SPLIT == kSplitA || SPLIT == kSplitA3)
              umma_bf16(d_tmem, sdesc_k_sw128(a1 + kk * 32), sdesc_k_sw128(b0 + kk * 32), idesc, 1);
            if (SPLIT == kSplitA3)
              umma_bf16(d_tmem, sdesc_k_sw128(a2 + kk * 32), sdesc_k_sw128(b0 + kk * 32), idesc, 1);
#pragma unroll
            for (int u = 1; u < MPI; ++u)
              if (u < mc)
                umma_bf16(d_tmem + u * kCols, sdesc_k_sw128(a0 + u * L::kAtile + kk * 32), sdesc_k_sw128(b0 + kk * 32),
                          idesc, (kb != kb_begin || kk != 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      if (ok) umma_commit(&acc_full[acc]);
    }
    if (!ok) {
      atomicExch(err, kDevTimeoutMma);
      *abort_flag = 1;
    }
    // wait for every MMA issued by this thread before TMEM is released
    umma_commit(drain);
    mbar_drain(drain, 0);
  } else if (W8 && warp >= 6) {
    // ---------------- converters (W8): FP8 tile -> bf16 tile in shared memory, laid out
    // with the 128-byte swizzle the MMA's descriptor expects. Warp 6 + w takes rows
    // 32 (w % 4) .. + 31 (one per lane) and k values 32 (w / 4) .. + 31 of the stage's 64.
    if constexpr (W8) {
      static_assert(MPI == 1, "W8: one weight tile per item");
      const int cw = warp - 6;
      const int q = warp & 3;
      const int r = q * 32 + lane;
      const int kh = cw >> 2;                       // which 32 k values
      const int ncb = sched.exp_ncb;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j) {
        const Tile t = sched.tile(j);
        // the scales of this warp's rows for the whole tile, one column block per lane
        // (two registers: blocks lane and lane + 32), fetched once and shuffled per k block
        const float sc_lo = lane < ncb ? ldexpf(1.0f, sched.exponent(t, 0, r, 2 * lane)) : 1.0f;
        const float sc_hi = lane + 32 < ncb ? ldexpf(1.0f, sched.exponent(t, 0, r, 2 * (lane + 32))) : 1.0f;
        for (int kb = kb_begin; kb < kb_end; ++kb) {
          if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, abort_flag))) { ok = false; break; }
          // the FP8 tile was stored with the 64-byte swizzle: 16-byte chunk c of row r sits
          // at chunk c ^ ((r >> 1) & 3) of its 64-byte row
          const uint8_t* row = sA + stage * L::kA + r * 64;
          uint4 v[2];
#pragma unroll
          for (int c = 0; c < 2; ++c)
            v[c] = *reinterpret_cast<const uint4*>(row + (((2 * kh + c) ^ ((r >> 1) & 3)) << 4));
          const int cb = kb >> 1;
          const float sc = __shfl_sync(0xffffffffu, cb < 32 ? sc_lo : sc_hi, cb & 31);
          uint32_t o[16];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              o[c * 8 + 2 * i] = e4m3x2_to_bf16x2((uint16_t)(w[i] & 0xFFFFu), sc);
              o[c * 8 + 2 * i + 1] = e4m3x2_to_bf16x2((uint16_t)(w[i] >> 16), sc);
            }
          }
          // 16-byte chunk c (8 k values) of row r goes to chunk c ^ (r & 7) of its 128-byte row
          uint8_t* out_row = smem + L::kOffAbf + stage * L::kAbf + r * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = kh * 4 + i;
            *reinterpret_cast<uint4*>(out_row + ((c ^ (r & 7)) << 4)) =
                make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          }
          fence_proxy_async_smem();   // the writes above are read by the tensor core
          mbar_arrive(&conv_full[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        atomicExch(err, kDevTimeoutProducer);
        *abort_flag = 1;
      }
    }
  } else if (warp >= 2) {
    // ---------------- epilogue
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;            // accumulator row owned by this thread
    for (int j = 0; j < ntiles; ++j) {
      const int acc = j % ACC_BUFS;
      const uint32_t acc_phase = (j / ACC_BUFS) & 1;
      const bool got = mbar_wait(&acc_full[acc], acc_phase, abort_flag);
      if (!epi_all(got)) {
        if (!got) atomicExch(err, kDevTimeoutEpilogue);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const Tile t0 = sched.tile(j);
      bool aborted = false;
      for (int u = 0; u < t0.m_count; ++u) {   // the item's m tiles, 128 rows apart
        Tile t = t0;
        t.mt += u;
        t.a_row += u * 128;
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (acc * MPI + u) * kCols;
        if constexpr (SPLIT == kSplitB) {
          // D = D_hi + D_lo, into the first columns the epilogue reads (the lo half starts
          // at the tile's column count: BN, or n16 for a dynamic-width tile)
          const int ncols = tile_cols<BN>(t);
#pragma unroll 1
          for (int c = 0; c < ncols; c += 16) {
            float hi[16], lo[16];
            tmem_ld16(taddr + c, hi);
            tmem_ld16(taddr + ncols + c, lo);
#pragma unroll
            for (int i = 0; i < 16; ++i) hi[i] += lo[i];
            tmem_st16(taddr + c, hi);
          }
        }
        if constexpr (KS > 1) {
          if (!splitk_reduce<BN, KS>(krank, taddr, r, smem, peer_ready, abort_flag, err)) {
            *abort_flag = 1;
            aborted = true;
            break;
          }
        }
        if (krank == 0) epi(t, taddr, r, epi_smem);
      }
      if (aborted) break;
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (KS > 1) cluster_sync();   // no CTA leaves while rank 0 may still read its shared memory
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ======================================================================== epilogues

// Plain fp32 store of D (used by the GEMM unit entry point).
template <int BN>
struct EpiStoreF32 {
  static constexpr int kSmemBytes = 0;
  float* out;
  int ldo;
  int N;
  long part_stride = 0;   // DensePartKSched: partial sum t.ks goes to out + t.ks * part_stride
  DLLM_DEV void operator()(const Tile& t, uint32_t taddr, int r, uint8_t*) const {
    const long row = t.a_row + r;
    float* out = this->out + t.ks * part_stride;
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      tmem_ld16(taddr + c, v);
      if (r < t.m_valid) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          int col = t.b_row + c + i;
          if (col < N) out[row * ldo + col] = v[i];
        }
      }
    }
  }
};

// Fused QKV epilogue: tile = one head (BN = head_dim) of the concatenated [Q | K | V]
// projection. Q and K get RoPE (rotate-half pairs (i, i + hd/2)); Q goes to the query
// buffer, K and V to the layer's KV cache at the token's absolute position.
template <int HD>
struct EpiQKV {
  static constexpr int kSmemBytes = 0;
  bf16_t* q;            // [T][H][HD]
  bf16_t* kc;           // layer cache [slots][Hkv][max_ctx][HD]
  bf16_t* vc;
  const float* rope_cos;   // [max_ctx][HD/2]
  const float* rope_sin;
  const int* pos0;      // per request: absolute position of its first token
  const int* slot;      // per request: KV slot
  int tok_per_req, H, Hkv, max_ctx;
  DLLM_DEV void operator()(const Tile& t, uint32_t taddr, int r, uint8_t*) const {
    constexpr int HALF = HD / 2;
    const int tok = t.a_row + r;
    const bool valid = r < t.m_valid;
    const int hh = t.nt;
    int b = 0, pos = 0;
    if (valid) {
      b = tok / tok_per_req;
      pos = pos0[b] + (tok - b * tok_per_req);
    }
    bf16_t* dst;
    if (hh < H) dst = q + ((long)tok * H + hh) * HD;
    else if (hh < H + Hkv) dst = kc + (((long)slot[b] * Hkv + (hh - H)) * max_ctx + pos) * HD;
    else dst = vc + (((long)slot[b] * Hkv + (hh - H - Hkv)) * max_ctx + pos) * HD;
    if (hh < H + Hkv) {
      static_assert(HALF % 8 == 0, "RoPE in 8-pair chunks");
      // four 8-pair chunks at a time: their cos / sin loads are issued together, ahead of
      // the TMEM reads, instead of one dependent global load per chunk
#pragma unroll 1
      for (int c0 = 0; c0 < HALF; c0 += 32) {
        float4 cs[4][2], sn[4][2];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = c0 + 8 * q;
          if (c < HALF && valid) {
            const float4* pc = reinterpret_cast<const float4*>(rope_cos + (long)pos * HALF + c);
            const float4* ps = reinterpret_cast<const float4*>(rope_sin + (long)pos * HALF + c);
            cs[q][0] = pc[0];
            cs[q][1] = pc[1];
            sn[q][0] = ps[0];
            sn[q][1] = ps[1];
          } else {
            cs[q][0] = cs[q][1] = sn[q][0] = sn[q][1] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = c0 + 8 * q;
          if (c >= HALF) break;   // warp-uniform
          float a[8], bb[8];
          tmem_ld8(taddr + c, a);
          tmem_ld8(taddr + c + HALF, bb);
          if (valid) {
            const float cv[8] = {cs[q][0].x, cs[q][0].y, cs[q][0].z, cs[q][0].w,
                                 cs[q][1].x, cs[q][1].y, cs[q][1].z, cs[q][1].w};
            const float sv[8] = {sn[q][0].x, sn[q][0].y, sn[q][0].z, sn[q][0].w,
                                 sn[q][1].x, sn[q][1].y, sn[q][1].z, sn[q][1].w};
            uint32_t lo[4], hi[4];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
              lo[i / 2] = pack_bf16x2(a[i] * cv[i] - bb[i] * sv[i], a[i + 1] * cv[i + 1] - bb[i + 1] * sv[i + 1]);
              hi[i / 2] = pack_bf16x2(bb[i] * cv[i] + a[i] * sv[i], bb[i + 1] * cv[i + 1] + a[i + 1] * sv[i + 1]);
            }
            *reinterpret_cast<uint4*>(dst + c) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            *reinterpret_cast<uint4*>(dst + c + HALF) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          }
        }
      }
    } else {
#pragma unroll 1
      for (int c = 0; c < HD; c += 8) {
        float a[8];
        tmem_ld8(taddr + c, a);
        if (valid) {
          *reinterpret_cast<uint4*>(dst + c) = make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]),
                                                          pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7]));
        }
      }
    }
  }
};

// Grouped gate/up epilogue: accumulator rows 0..63 are gate features 64*mt + r, rows
// 64..127 the matching up features; columns are the chunk's tokens. The up half goes
// through shared memory; h = silu(g) * u is written as the (hi, lo) bf16 pair that the
// down GEMM consumes.
template <int BN>
struct EpiSwiGLU {
  static constexpr int kSmemBytes = 16 * 65 * 4;
  bf16_t* h;     // [slots][F], hi part
  bf16_t* h_lo;  // [slots][F], lo part
  int F;
  DLLM_DEV void operator()(const Tile& t, uint32_t taddr, int r, uint8_t* smem) const {
    float* us = reinterpret_cast<float*>(smem);
    const int f = t.mt * 64 + (r & 63);
    const int ncols = tile_cols<BN>(t);
#pragma unroll 1
    for (int c = 0; c < ncols; c += 16) {
      float v[16];
      tmem_ld16(taddr + c, v);
      if (r >= 64) {
#pragma unroll
        for (int i = 0; i < 16; ++i) us[i * 65 + (r - 64)] = v[i];
      }
      epi_bar_sync();
      if (r < 64) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int n = c + i;
          if (n < t.n_valid) {
            const float g = v[i];
            const float u = us[i * 65 + r];
            const float hv = g / (1.0f + __expf(-g)) * u;
            const bf16_t hi = f32_to_bf16(hv);
            const long o = (long)(t.b_row + n) * F + f;
            h[o] = hi;
            h_lo[o] = f32_to_bf16(hv - bf16_to_f32(hi));
          }
        }
      }
      epi_bar_sync();
    }
  }
};

// x[token][feature] += D with the operands swapped (the attention output projection run
// as Wo x ao^T): accumulator rows are output features a_row + r, columns the chunk's
// tokens b_row + c. Lanes hold consecutive features, so each column's read-modify-write
// of x is one coalesced 128-byte access per warp.
template <int BN>
struct EpiResidualT {
  static constexpr int kSmemBytes = 0;
  float* x;
  int ldx;
  int T;   // token rows
  DLLM_DEV void operator()(const Tile& t, uint32_t taddr, int r, uint8_t*) const {
    const int f = t.a_row + r;
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 16) {
      float old[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int tok = t.b_row + c0 + i;
        old[i] = (tok < T && r < t.m_valid) ? x[(long)tok * ldx + f] : 0.f;
      }
      float v[16];
      tmem_ld16(taddr + c0, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int tok = t.b_row + c0 + i;
        if (tok < T && r < t.m_valid) x[(long)tok * ldx + f] = old[i] + v[i];
      }
    }
  }
};

// Split-K partial of the swapped-operand O projection: partial t.ks of D^T, stored as
// part[t.ks][token][feature] in fp32 (coalesced across the feature lanes like
// EpiResidualT); the RMSNorm kernel that follows adds the partials into x in slice order.
template <int BN>
struct EpiPartialT {
  static constexpr int kSmemBytes = 0;
  float* part;
  int ldp;      // features per row (d)
  int T;        // token rows
  long stride;  // elements per partial (T_max * d)
  DLLM_DEV void operator()(const Tile& t, uint32_t taddr, int r, uint8_t*) const {
    const int f = t.a_row + r;
    float* p = part + t.ks * stride;
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 16) {
      float v[16];
      tmem_ld16(taddr + c0, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int tok = t.b_row + c0 + i;
        if (tok < T && r < t.m_valid) p[(long)tok * ldp + f] = v[i];
      }
    }
  }
};

// Grouped down epilogue: accumulator rows are output features 128*mt + r, columns the
// chunk's tokens; o[slot][feature] in fp32 for the combine.
template <int BN>
struct EpiDown {
  static constexpr int kSmemBytes = 0;
  float* o;      // [slots][d]
  int d;
  DLLM_DEV void operator()(const Tile& t, uint32_t taddr, int r, uint8_t*) const {
    const int dd = t.mt * 128 + r;
    const int ncols = tile_cols<BN>(t);
#pragma unroll 1
    for (int c = 0; c < ncols; c += 16) {
      float v[16];
      tmem_ld16(taddr + c, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int n = c + i;
        if (n < t.n_valid) o[(long)(t.b_row + n) * d + dd] = v[i];
      }
    }
  }
};

// LM-head epilogue: per row, over this tile's BN vocabulary columns, the running
// maximum logit, its (lowest) token id and sum exp(l - max), with [MASK] left out.
// Logits never leave the SM; a merge kernel combines the per-tile partials.
template <int BN>
struct EpiLMHead {
  static constexpr int kSmemBytes = 0;
  float* part_m;      // [rows][n_vtiles]
  float* part_s;
  int* part_i;
  int n_vtiles;
  int mask_id;
  DLLM_DEV void operator()(const Tile& t, uint32_t taddr, int r, uint8_t*) const {
    constexpr float kLog2e = 1.4426950408889634f;
    float m = -INFINITY, s = 0.f;
    int idx = 0;
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      tmem_ld16(taddr + c, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int col = t.b_row + c + i;
        const float l = v[i];
        if (col == mask_id) continue;
        if (l > m) {
          s = s * exp2f((m - l) * kLog2e) + 1.0f;
          m = l;
          idx = col;
        } else {
          s += exp2f((l - m) * kLog2e);
        }
      }
    }
    if (r < t.m_valid) {
      const long o = (long)(t.a_row + r) * n_vtiles + t.nt;
      part_m[o] = m;
      part_s[o] = s;
      part_i[o] = idx;
    }
  }
};

}  // namespace dllm
