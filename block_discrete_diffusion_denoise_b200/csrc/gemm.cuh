// Persistent, warp-specialised tcgen05 GEMM for sm_100a.
//
//   D[m, n] = sum_k A[m, k] * B[n, k]        (A, B bf16 K-major; D fp32 in TMEM)
//
// One CTA per SM.  Warp 0 (one lane) loads the A operand and warp 6 (one
// lane) the B operand of every stage of one ring of shared-memory stages (6
// for MOE, 4 otherwise) with TMA, warp 1 (one lane) issues tcgen05.mma into
// one of two TMEM accumulators (128 lanes x 128 or 256 fp32 columns each),
// warps 2..5 drain the other accumulator through the epilogue.  All waits are
// bounded.
//
// Three launch modes share the pipeline:
//   DENSE   A = weight rows (output features), B = up to 256 tokens; split-K
//           partials out[split][token][feature] fp32, summed in split order by
//           the consumer kernel (deterministic, no atomics).  Static tiles.
//   MOE     one launch for all experts of a layer, routed and shared: first the
//           gate/up tiles (A = 64 gate rows stacked on the same 64 up rows, B =
//           the expert's tokens; the epilogue forms SiLU(gate) * up and stores
//           bf16 hidden rows), then the down tiles (A = 128 rows of the down
//           projection, B = hidden rows; fp32 output rows in the expert's
//           region).  Every CTA derives the tile list from the per-expert row
//           counts in shared memory; tiles are claimed from an atomic counter
//           in list order; a down tile waits until every gate/up tile of its
//           token chunk has published its hidden rows.  Every claimed tile's
//           dependencies were claimed earlier by running CTAs and depend on
//           nothing, so the wait always ends.
//   LMHEAD  A = two 128-token tiles (each vocabulary block is loaded once for
//           256 tokens), B = 128 vocabulary rows of the tied embedding; the
//           epilogue keeps, per token, the running top-2 logits, the argmax,
//           the sum of 2^x and the sum of 2^x * x (for the entropy), and
//           writes one 16-byte partial (+ 4 bytes) per (vocabulary tile,
//           token) — the logits never reach memory.
#pragma once

#include "common.cuh"

namespace dg {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 64;
constexpr int GEMM_BN = 128;                         // accumulator columns; dense / LM-head tile width
constexpr int GEMM_A_BYTES = GEMM_BM * GEMM_BK * 2;  // 16 KB
// warp 0: A producer, warp 1: MMA issuer, warps 2-5: epilogue, warp 6: B producer
constexpr int GEMM_THREADS = 224;
constexpr int GEMM_B_WARP = 6;
// epilogue staging: gate values of one 32-column chunk (64 x 33) or one
// 32 x 128 fp32 block on its way to global memory
constexpr int GEMM_XCHG_FLOATS = 2 * 32 * GEMM_BM;
constexpr int GEMM_SCHED = 4;                        // claimed-tile ring
constexpr int MOE_CHUNK_ROWS = 128;                  // tokens per expert tile

enum GemmMode : int { GEMM_DENSE = 0, GEMM_MOE = 1, GEMM_LMHEAD = 3 };

constexpr int DENSE_BN = 256;                        // tokens per dense tile: each weight tile streamed once
constexpr int MOE_MAX_EXPERTS = 256;                 // routed experts (+1 shared group) the tile tables hold
// MOE tile tables in shared memory: chunk offsets [E + 2] and group rows [E + 1], 16-bit
constexpr int MOE_TABLE_BYTES = ((MOE_MAX_EXPERTS + 2) + (MOE_MAX_EXPERTS + 1)) * 2 + 32;

// Stage ring depth (16 KB of A plus the B rows of one k-step per stage).
// Two producers fill each stage: warp 0 its A half, warp 6 its B half (the
// stage's full barrier takes two arrivals), so a wait that holds back one
// operand (a down tile's dependency) does not stop the other's loads.
template <int MODE>
constexpr int gemm_stages() {
  return MODE == GEMM_MOE ? 6 : 4;
}
// 128-row A tiles per CTA tile: the LM head takes two token tiles (256
// tokens) per vocabulary block, so each 128-row block of the embedding is
// loaded once for both and L2 carries a third less operand traffic
template <int MODE>
constexpr int gemm_halves() {
  return MODE == GEMM_LMHEAD ? 2 : 1;
}
template <int MODE>
constexpr int gemm_a_bytes() {
  return GEMM_A_BYTES * gemm_halves<MODE>();
}
// LM-head tiles per vocabulary block: pairs of 128-token tiles
__host__ __device__ constexpr int lmhead_mpairs(int n_mtiles) { return (n_mtiles + 1) / 2; }
// rows of B one stage holds
template <int MODE>
constexpr int gemm_b_rows() {
  return MODE == GEMM_MOE ? MOE_CHUNK_ROWS : (MODE == GEMM_DENSE ? DENSE_BN : GEMM_BN);
}
template <int MODE>
constexpr int gemm_b_bytes() {
  return gemm_b_rows<MODE>() * GEMM_BK * 2;
}
// fp32 columns of one of the two TMEM accumulators (a power of two)
template <int MODE>
constexpr int gemm_acc_cols() {
  return gemm_b_rows<MODE>() > 128 ? 256 : 128;
}
template <int MODE>
constexpr int gemm_smem_bytes() {
  return 1024 + gemm_stages<MODE>() * (gemm_a_bytes<MODE>() + gemm_b_bytes<MODE>()) + GEMM_XCHG_FLOATS * 4 + 512 +
         (MODE == GEMM_MOE ? MOE_TABLE_BYTES : 0);
}

enum TileKind : int { KIND_DENSE = 0, KIND_GATEUP = 1, KIND_DOWN = 2, KIND_LMHEAD = 3 };

struct GemmParams {
  CUtensorMap a_map[2];   // DENSE/LMHEAD: [0]; MOE gate/up routed: [0] w_gate, [1] w_up
  CUtensorMap as_map[2];  // MOE gate/up shared expert: [0] ws_gate, [1] ws_up
  CUtensorMap b_map;      // DENSE: tokens; LMHEAD: embed; MOE gate/up routed: gathered rows
  CUtensorMap bs_map;     // MOE gate/up shared: normed tokens
  CUtensorMap d_map;      // MOE down routed A: w_down
  CUtensorMap ds_map;     // MOE down shared A: ws_down
  CUtensorMap h_map;      // MOE down routed B: routed hidden rows
  CUtensorMap hs_map;     // MOE down shared B: shared hidden rows
  // MOE: the same B tensors in 64-row boxes; whole 64-row groups go in one
  // copy each, the rest in b_box_rows boxes (fewer copies measured faster;
  // 128-row boxes measured slower than two 64-row ones)
  CUtensorMap b_mid_map, bs_mid_map, h_mid_map, hs_mid_map;
  CUtensorMap out_map;    // DENSE: fp32 partials as 3-D (M, T, splits), box (128, 64, 1); see use_tma_store
  int b_box_rows;         // rows per B box (16 MOE, 64 DENSE, 128 LM head)
  int b_mid_rows;         // 0 = none (64 MOE)
  int M;                  // DENSE: output features; LMHEAD: tokens
  int T;                  // DENSE: tokens
  int k_steps;            // K / 64 (DENSE, LMHEAD)
  int splits;             // DENSE split-K
  int n_tiles_n;          // DENSE token tiles
  int bn;                 // DENSE token tile
  int n_mtiles;           // LMHEAD token tiles
  int tiles_static;       // DENSE / LMHEAD tile count
  int use_tma_store;      // DENSE: a CTA's last tile is staged in the operand ring and stored by TMA
  int a_mn_major;         // DENSE: A stored [K][M] (M contiguous), read as two [64 k][64 m] boxes per stage
  // LMHEAD, probability mode: write p = 2^(x - lse2[token]) as bf16 [T][V]
  // (via p_map, box 64 x 128, 128-byte swizzle) instead of the statistics
  const float* lse2;      // per-token log-sum-exp in log2 units, or NULL (statistics mode)
  CUtensorMap p_map;
  // DENSE, MOE: claimed tiles
  int* work;              // [0] claim counter, [1] exit counter; zero at launch, reset by the last CTA
  // MOE
  int* expert_rows;       // [E] rows routed to each expert (zeroed by the last CTA out)
  int region;             // rows per expert region of the routed buffers
  int* chunk_done;        // finished gate/up tiles per token chunk, zero at launch (zeroed by the last CTA)
  int n_groups_routed;    // E; group == n_groups_routed is the shared expert (its T rows are the tokens)
  int F, Fs, d;
  float* out_f32;         // DENSE partials [splits][T][M]; MOE down output rows [.][out_ld]
  int out_ld;
  int shared_row_base;    // MOE down: output row of shared-expert token 0
  uint16_t* h_out;        // MOE routed hidden [rows][F]
  uint16_t* hs_out;       // MOE shared hidden [tokens][Fs]
  float4* lm_part;        // LMHEAD partials [vocab tiles][M]: {max, argmax, second max, sum 2^(x - max)}
  float* lm_s1;           // LMHEAD [vocab tiles][M]: sum 2^(x - max) * x (entropy), or NULL
  float logit_scale_log2; // LMHEAD: log2(e) / temperature
  DevErr err;
};

struct GemmTile {
  const CUtensorMap* a0;
  const CUtensorMap* a1;  // second 64-row A box (gate/up) or nullptr
  int a_row;
  const CUtensorMap* b;
  const CUtensorMap* b_mid;  // the same tensor in b_mid_rows boxes
  int b_row;
  int n;      // valid columns
  int nmma;   // MMA N (multiple of 16, <= 128)
  int k0, nk;
  int split, group, blk, chunk;
  int kind;
  int halves;     // 128-row A tiles (LMHEAD: 1 or 2 token tiles)
  bool shared;
  bool a_stream;  // A is read once (evict-first)
};

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

// rec: the MOE tile record (from the tile list); n_gu: number of gate/up tiles
template <int MODE>
__device__ __forceinline__ void decode_tile(const GemmParams& p, int tile, int4 rec, int n_gu, GemmTile& t) {
  t.chunk = 0;
  t.shared = false;
  t.halves = 1;
  if constexpr (MODE == GEMM_DENSE) {
    const int nt = tile % p.n_tiles_n;
    const int rest = tile / p.n_tiles_n;
    t.split = rest % p.splits;
    const int mt = rest / p.splits;
    t.kind = KIND_DENSE;
    t.a0 = &p.a_map[0];
    t.a1 = nullptr;
    t.a_row = mt * GEMM_BM;
    t.b = &p.b_map;
    t.b_mid = &p.b_mid_map;
    t.b_row = nt * p.bn;
    t.n = min(p.bn, p.T - t.b_row);
    t.nmma = round16(t.n);
    t.k0 = (t.split * p.k_steps) / p.splits;
    t.nk = ((t.split + 1) * p.k_steps) / p.splits - t.k0;
    t.group = 0;
    t.blk = mt;
    t.a_stream = p.n_tiles_n == 1;
  } else if constexpr (MODE == GEMM_LMHEAD) {
    const int np = lmhead_mpairs(p.n_mtiles);
    const int vt = tile / np;
    const int mp = tile % np;
    t.kind = KIND_LMHEAD;
    t.a0 = &p.a_map[0];
    t.a1 = nullptr;
    t.a_row = mp * 2 * GEMM_BM;
    t.halves = min(2, p.n_mtiles - 2 * mp);
    t.b = &p.b_map;
    t.b_mid = &p.b_mid_map;
    t.b_row = vt * GEMM_BN;
    t.n = GEMM_BN;
    t.nmma = GEMM_BN;
    t.k0 = 0;
    t.nk = p.k_steps;
    t.split = 0;
    t.group = vt;
    t.blk = mp;
    t.a_stream = false;
  } else {
    const int4 e = rec;
    const bool down = tile >= n_gu;
    t.group = e.x & 0xffff;
    t.blk = e.x >> 16;
    t.chunk = e.y;
    t.b_row = e.z;
    t.n = e.w;
    t.nmma = round16(e.w);
    t.k0 = 0;
    t.split = 0;
    t.shared = t.group == p.n_groups_routed;
    t.a_stream = !t.shared;
    if (!down) {
      t.kind = KIND_GATEUP;
      t.a0 = t.shared ? &p.as_map[0] : &p.a_map[0];
      t.a1 = t.shared ? &p.as_map[1] : &p.a_map[1];
      t.a_row = (t.shared ? 0 : t.group * p.F) + t.blk * 64;
      t.b = t.shared ? &p.bs_map : &p.b_map;
      t.b_mid = t.shared ? &p.bs_mid_map : &p.b_mid_map;
      t.nk = p.d / GEMM_BK;
    } else {
      t.kind = KIND_DOWN;
      t.a0 = t.shared ? &p.ds_map : &p.d_map;
      t.a1 = nullptr;
      t.a_row = (t.shared ? 0 : t.group * p.d) + t.blk * GEMM_BM;
      t.b = t.shared ? &p.hs_map : &p.h_map;
      t.b_mid = t.shared ? &p.hs_mid_map : &p.h_mid_map;
      t.nk = (t.shared ? p.Fs : p.F) / GEMM_BK;
    }
  }
}

// MOE tile list, derived from the row counts.  Groups g = 0 (shared expert,
// T rows) and g = 1 + e (routed expert e); group g has nch_g = ceil(rows_g /
// MOE_CHUNK_ROWS) token chunks; ch_off[g] = sum of nch over the groups before
// g (ch_off[G] = all chunks).  Gate/up tiles first: the shared group's Fs/64
// blocks x nch_0 chunks, then each routed group's F/64 blocks x nch_g chunks;
// then the down tiles: each group's d/128 blocks x nch_g chunks.  Within a
// group the order is block-major, so re-reads of a weight block by its chunks
// hit L2.  Record: {group (E = shared) | block << 16, chunk id, first row,
// rows}.
struct MoeTables {
  const uint16_t* ch_off;  // [G + 1]
  const uint16_t* rows;    // [G]
  int G;                   // E + 1 groups
  int n_gu, n_dn;
};

__device__ __forceinline__ int moe_upper(const uint16_t* a, int n, int q) {  // first i in [0, n) with a[i] > q
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (static_cast<int>(a[mid]) > q) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

__device__ __forceinline__ int4 moe_record(const GemmParams& p, const MoeTables& tb, int t) {
  const int mb_s = p.Fs / 64, mb_r = p.F / 64, mb_dn = p.d / GEMM_BM;
  const int nch_s = tb.ch_off[1];
  int g, local;
  if (t < tb.n_gu) {
    if (t < nch_s * mb_s) {
      g = 0;
      local = t;
    } else {
      const int tp = t - nch_s * mb_s;
      g = moe_upper(tb.ch_off, tb.G + 1, tp / mb_r + nch_s) - 1;
      local = tp - (static_cast<int>(tb.ch_off[g]) - nch_s) * mb_r;
    }
  } else {
    const int tp = t - tb.n_gu;
    g = moe_upper(tb.ch_off, tb.G + 1, tp / mb_dn) - 1;
    local = tp - static_cast<int>(tb.ch_off[g]) * mb_dn;
  }
  const int nch = tb.ch_off[g + 1] - tb.ch_off[g];
  const int blk = local / nch, ch = local % nch;
  const int first = (g == 0 ? 0 : (g - 1) * p.region) + ch * MOE_CHUNK_ROWS;
  return make_int4((g == 0 ? p.n_groups_routed : g - 1) | (blk << 16), tb.ch_off[g] + ch, first,
                   min(MOE_CHUNK_ROWS, static_cast<int>(tb.rows[g]) - ch * MOE_CHUNK_ROWS));
}

// exclusive scan of one value per thread over the whole block (blockDim.x a
// multiple of 32); tmp >= 32 ints; every thread receives the total
__device__ __forceinline__ int block_excl_scan(int v, int* tmp, int& total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  int base = 0;
  total = 0;
  for (int w = 0; w < nw; ++w) {
    const int t = tmp[w];
    if (w < warp) base += t;
    total += t;
  }
  __syncthreads();
  return base + x - v;
}

template <int MODE>
__device__ __forceinline__ int tile_total(const GemmParams& p, const MoeTables& tb) {
  if constexpr (MODE == GEMM_MOE) return tb.n_gu + tb.n_dn;
  return p.tiles_static;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* ptr) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_gpu_add(int* ptr, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}

// Wait (bounded) until every gate/up tile of `chunk` has published its rows.
__device__ __forceinline__ bool wait_chunk_ready(const GemmParams& p, const GemmTile& t) {
  const int need = (t.shared ? p.Fs : p.F) / 64;
  const int* flag = p.chunk_done + t.chunk;
  if (ld_acquire_gpu(flag) < need) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(flag) < need) {
      if (globaltimer_ns() - t0 > p.err.limit_ns) {
        raise_error(p.err, ERR_TIMEOUT);
        return false;
      }
      __nanosleep(64);
    }
  }
  fence_proxy_async_global();
  return true;
}

// Store a 128-column x 32-row fp32 block held one column per epilogue thread
// (thread `col` has v[i] = element (row i, column col)) to dst[i * ld + col]
// for i < nrows, col < ncols.  The block is transposed through shared memory
// so each warp instruction writes 512 contiguous bytes as 16-byte vectors;
// all eight shared-memory reads are issued before the first global store.
// Called by all 128 epilogue threads; dst and ld keep 16-byte alignment.
// Successive calls within a tile alternate between the two halves of the
// exchange area: the next call's barrier orders this call's reads before
// its half is written again, and the barriers at the start of every tile
// do the same across tiles.
__device__ __forceinline__ void store_rows_via_smem(float* stage, const float* v, int col, int etid, float* dst,
                                                    int ld, int nrows, int ncols) {
  const uint32_t sb = smem_u32(stage);
#pragma unroll
  for (int i = 0; i < 32; ++i)
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(sb + (i * GEMM_BM + col) * 4), "f"(v[i]) : "memory");
  named_bar_sync(1, 128);
  float4 x[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int idx = etid + 128 * r;
    const int i = idx >> 5, c4 = (idx & 31) * 4;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(x[r].x), "=f"(x[r].y), "=f"(x[r].z), "=f"(x[r].w)
                 : "r"(sb + (i * GEMM_BM + c4) * 4)
                 : "memory");
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int idx = etid + 128 * r;
    const int i = idx >> 5, c4 = (idx & 31) * 4;
    if (i < nrows && c4 < ncols) {
      float* d = dst + static_cast<size_t>(i) * ld + c4;
      if (c4 + 4 <= ncols) {
        asm volatile("st.global.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(__cvta_generic_to_global(d)), "f"(x[r].x),
                     "f"(x[r].y), "f"(x[r].z), "f"(x[r].w)
                     : "memory");
      } else {
        d[0] = x[r].x;
        if (c4 + 1 < ncols) d[1] = x[r].y;
        if (c4 + 2 < ncols) d[2] = x[r].z;
      }
    }
  }
}

template <int MODE>
constexpr bool claims_tiles() {
  return MODE == GEMM_MOE;
}

template <int MODE>
__global__ void __launch_bounds__(GEMM_THREADS, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  DG_TIMELINE_SCOPE(TLK_GEMM + MODE);
  constexpr int STAGES = gemm_stages<MODE>();
  constexpr int A_BYTES = gemm_a_bytes<MODE>();
  constexpr int HALVES = gemm_halves<MODE>();
  constexpr int B_BYTES = gemm_b_bytes<MODE>();
  static_assert(gemm_smem_bytes<MODE>() <= 232448, "shared memory per CTA");
  static_assert((2 * STAGES + 5 + 2 * GEMM_SCHED) * 8 + GEMM_SCHED * 20 + 64 <= 512, "barrier area");
  constexpr int ACC_COLS = gemm_acc_cols<MODE>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  float* xchg = reinterpret_cast<float*>(sB + STAGES * B_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(xchg + GEMM_XCHG_FLOATS);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* sched_full = drain + 1;
  uint64_t* sched_empty = sched_full + GEMM_SCHED;
  int4* sched_rec = reinterpret_cast<int4*>((reinterpret_cast<uintptr_t>(sched_empty + GEMM_SCHED) + 15) &
                                            ~uintptr_t(15));
  int* sched = reinterpret_cast<int*>(sched_rec + GEMM_SCHED);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sched + GEMM_SCHED);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* scan_tmp = reinterpret_cast<int*>(tmem_holder + 4);           // 8 ints
  uint16_t* tb_ch_off = reinterpret_cast<uint16_t*>(xchg + GEMM_XCHG_FLOATS) + 256;  // after the 512-byte tail
  uint16_t* tb_rows = tb_ch_off + MOE_MAX_EXPERTS + 2;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // the operand descriptors are fetched while the CTA sets up
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&p.a_map[0]);
    tma_prefetch_desc(&p.b_map);
  }
  // barriers and TMEM first: their latency overlaps the tile-table loads
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 2);  // the A and the B producer
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    for (int s = 0; s < GEMM_SCHED; ++s) {
      mbar_init(&sched_full[s], 1);
      mbar_init(&sched_empty[s], 3);  // B producer + MMA issuer + epilogue leader
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 2 * ACC_COLS * HALVES);
    tmem_relinquish();
  }
  MoeTables tb{tb_ch_off, tb_rows, 0, 0, 0};
  if constexpr (MODE == GEMM_MOE) {
    // tile tables from the row counts (two groups per thread, G <= 2 * GEMM_THREADS)
    const int G = p.n_groups_routed + 1;
    int nch2[2], rows2[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int g = 2 * threadIdx.x + h;
      rows2[h] = g == 0 ? p.T : (g < G ? p.expert_rows[g - 1] : 0);
      nch2[h] = (rows2[h] + MOE_CHUNK_ROWS - 1) / MOE_CHUNK_ROWS;
    }
    int total;
    const int base = block_excl_scan(nch2[0] + nch2[1], scan_tmp, total);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int g = 2 * threadIdx.x + h;
      if (g < G) {
        tb_rows[g] = static_cast<uint16_t>(rows2[h]);
        tb_ch_off[g] = static_cast<uint16_t>(base + (h ? nch2[0] : 0));
      }
    }
    if (threadIdx.x == 0) tb_ch_off[G] = static_cast<uint16_t>(total);
    __syncthreads();
    const int nch_s = tb_ch_off[1];
    tb.G = G;
    tb.n_gu = nch_s * (p.Fs / 64) + (total - nch_s) * (p.F / 64);
    tb.n_dn = total * (p.d / GEMM_BM);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int n_tiles = tile_total<MODE>(p, tb);
  const int n_gu = tb.n_gu;

  if (warp == 0) {
    if (lane == 0) {
      // --------------------------- TMA producer of A ---------------------------
      // Claims the tiles (MOE), publishes them to the other roles, and fills
      // the A half of each stage.
      tma_prefetch_desc(&p.a_map[0]);
      const uint64_t pol_first = policy_evict_first();
      const uint64_t pol_last = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_par = 0;
      int cur = -1, claim = 0;
      int4 cur_rec = make_int4(0, 0, 0, 0);
      if constexpr (claims_tiles<MODE>()) {
        // the first tile of every CTA is its own index; later tiles are
        // claimed from the counter, which numbers the tiles after those
        cur = blockIdx.x;
        if (cur < n_tiles) cur_rec = moe_record(p, tb, cur);
        claim = static_cast<int>(gridDim.x) + atomicAdd(p.work, 1);
      }
      for (int it = 0;; ++it) {
        int tile;
        int4 rec = make_int4(0, 0, 0, 0);
        int nxt = -1;
        int4 nxt_rec = make_int4(0, 0, 0, 0);
        if constexpr (claims_tiles<MODE>()) {
          if (cur >= n_tiles || *abort_flag) cur = -1;
          tile = cur;
          rec = cur_rec;
          const int slot = it % GEMM_SCHED;
          if (!mbar_wait(&sched_empty[slot], ((it / GEMM_SCHED) & 1) ^ 1, p.err)) {
            *abort_flag = 1;
            break;
          }
          sched[slot] = tile;
          sched_rec[slot] = rec;
          mbar_arrive(&sched_full[slot]);
          if (tile < 0) break;
        } else {
          tile = blockIdx.x + it * gridDim.x;
          if (tile >= n_tiles || *abort_flag) break;
        }
        GemmTile t;
        decode_tile<MODE>(p, tile, rec, n_gu, t);
        const uint64_t pol_a = t.a_stream ? pol_first : pol_last;
        for (int k = 0; k < t.nk; ++k) {
          if constexpr (claims_tiles<MODE>()) {
            // the next claim and its record are taken once this tile's first
            // loads are in flight (the claim's atomic was issued a tile
            // earlier, or at setup), so no global round trip sits between
            // tiles or before the first one
            if (k == min(2, t.nk - 1) && claim < n_tiles) {
              nxt = claim;
              nxt_rec = moe_record(p, tb, nxt);
              claim = static_cast<int>(gridDim.x) + atomicAdd(p.work, 1);
            }
          }
          if (!mbar_wait(&empty[stage], phase ^ 1, p.err)) {
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], GEMM_A_BYTES * t.halves);
          uint8_t* a = sA + stage * A_BYTES;
          const int kx = (t.k0 + k) * GEMM_BK;
          if (MODE == GEMM_DENSE && p.a_mn_major) {
            // A stored [K][M]: two boxes of 64 k-rows x 64 m-columns
            tma_load_2d(a, t.a0, &full[stage], t.a_row, kx, pol_a);
            tma_load_2d(a + GEMM_A_BYTES / 2, t.a0, &full[stage], t.a_row + 64, kx, pol_a);
          } else {
            tma_load_2d(a, t.a0, &full[stage], kx, t.a_row, pol_a);
            if (t.a1 != nullptr) tma_load_2d(a + GEMM_A_BYTES / 2, t.a1, &full[stage], kx, t.a_row, pol_a);
            if (HALVES > 1 && t.halves > 1)
              tma_load_2d(a + GEMM_A_BYTES, t.a0, &full[stage], kx, t.a_row + GEMM_BM, pol_a);
          }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (*abort_flag) break;
        if constexpr (claims_tiles<MODE>()) {
          cur = nxt;
          cur_rec = nxt_rec;
        }
      }
      // every copy this thread issued has landed before the CTA may exit
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1) mbar_wait(&full[s], (issued_par >> s) & 1, p.err);
    }
  } else if (warp == GEMM_B_WARP) {
    if (lane == 0) {
      // --------------------------- TMA producer of B ---------------------------
      // Follows the same tiles and fills the B half of each stage.  A down
      // tile's rows are the hidden rows its chunk's gate/up tiles publish, so
      // before its first B load this warp waits (bounded) for the chunk's
      // counter with acquire and orders the TMA reads after it with a proxy
      // fence; meanwhile the A producer keeps loading weights.
      tma_prefetch_desc(&p.b_map);
      const uint64_t pol_last = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_par = 0;
      for (int it = 0;; ++it) {
        int tile;
        int4 rec = make_int4(0, 0, 0, 0);
        if constexpr (claims_tiles<MODE>()) {
          const int slot = it % GEMM_SCHED;
          if (!mbar_wait(&sched_full[slot], (it / GEMM_SCHED) & 1, p.err)) {
            *abort_flag = 1;
            break;
          }
          tile = sched[slot];
          rec = sched_rec[slot];
          mbar_arrive(&sched_empty[slot]);
          if (tile < 0) break;
        } else {
          tile = blockIdx.x + it * gridDim.x;
          if (tile >= n_tiles) break;
        }
        if (*abort_flag) break;
        GemmTile t;
        decode_tile<MODE>(p, tile, rec, n_gu, t);
        if constexpr (MODE == GEMM_MOE) {
          if (t.kind == KIND_DOWN && !wait_chunk_ready(p, t)) {
            *abort_flag = 1;
            break;
          }
        }
        // B arrives in whole boxes (rows past nmma are loaded, zero-filled
        // past the tensor's end, and ignored by the MMA)
        const int b_rows = (t.nmma + p.b_box_rows - 1) / p.b_box_rows * p.b_box_rows;
        const uint32_t bytes = b_rows * GEMM_BK * 2;
        for (int k = 0; k < t.nk; ++k) {
          if (!mbar_wait(&empty[stage], phase ^ 1, p.err)) {
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], bytes);
          uint8_t* b = sB + stage * B_BYTES;
          const int kx = (t.k0 + k) * GEMM_BK;
          int r = 0;
          if (p.b_mid_rows > 0)
            for (; r + p.b_mid_rows <= t.nmma; r += p.b_mid_rows)
              tma_load_2d(b + r * (GEMM_BK * 2), t.b_mid, &full[stage], kx, t.b_row + r, pol_last);
          for (; r < t.nmma; r += p.b_box_rows)
            tma_load_2d(b + r * (GEMM_BK * 2), t.b, &full[stage], kx, t.b_row + r, pol_last);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (*abort_flag) break;
      }
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1) mbar_wait(&full[s], (issued_par >> s) & 1, p.err);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool aborted = false;
      for (int it = 0;; ++it) {
        int tile;
        int4 rec = make_int4(0, 0, 0, 0);
        if constexpr (claims_tiles<MODE>()) {
          const int slot = it % GEMM_SCHED;
          if (!mbar_wait(&sched_full[slot], (it / GEMM_SCHED) & 1, p.err)) {
            aborted = true;
            break;
          }
          tile = sched[slot];
          rec = sched_rec[slot];
          mbar_arrive(&sched_empty[slot]);
          if (tile < 0) break;
        } else {
          tile = blockIdx.x + it * gridDim.x;
          if (tile >= n_tiles) break;
        }
        if (*abort_flag) {
          aborted = true;
          break;
        }
        GemmTile t;
        decode_tile<MODE>(p, tile, rec, n_gu, t);
        const int acc = it & 1;
        const uint32_t acc_par = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_par ^ 1, p.err)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * ACC_COLS * HALVES;
        const bool a_mn = MODE == GEMM_DENSE && p.a_mn_major;
        const uint32_t idesc = umma_idesc_bf16(GEMM_BM, t.nmma) | (a_mn ? (1u << 15) : 0u);
        for (int k = 0; k < t.nk; ++k) {
          if (!mbar_wait(&full[stage], phase, p.err)) {
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint32_t a_at = smem_u32(sA + stage * A_BYTES);
          const uint64_t bd = umma_desc_sw128(smem_u32(sB + stage * B_BYTES));
          if (a_mn) {
            // MN-major A: 16 k-rows are 2048 bytes; the two 64-wide m blocks are GEMM_A_BYTES / 2 apart
#pragma unroll
            for (int kk = 0; kk < GEMM_BK / 16; ++kk)
              umma_bf16(d_tmem, umma_desc_sw128_mn(a_at + kk * 2048, GEMM_A_BYTES / 2), bd + 2 * kk, idesc,
                        (k | kk) != 0);
          } else {
            const uint64_t ad = umma_desc_sw128(a_at);
#pragma unroll
            for (int kk = 0; kk < GEMM_BK / 16; ++kk)
              umma_bf16(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (k | kk) != 0);
            if (HALVES > 1 && t.halves > 1) {
              // the second token tile against the same B (vocabulary) tile
              const uint64_t ad1 = umma_desc_sw128(a_at + GEMM_A_BYTES);
#pragma unroll
              for (int kk = 0; kk < GEMM_BK / 16; ++kk)
                umma_bf16(d_tmem + ACC_COLS, ad1 + 2 * kk, bd + 2 * kk, idesc, (k | kk) != 0);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (aborted) break;
        umma_commit(&tfull[acc]);
      }
      if (aborted) {
        *abort_flag = 1;
        umma_commit(drain);               // all issued MMAs finish before TMEM is freed
        mbar_wait(drain, 0, p.err);
      }
    }
  } else {
    // ------------------------------ epilogue (warps 2-5) -----------------------
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;       // tile row owned by this thread
    const int etid = threadIdx.x - 64;   // 0..127
    for (int it = 0;; ++it) {
      int tile = -1;
      int4 rec = make_int4(0, 0, 0, 0);
      bool ok = *abort_flag == 0;
      if constexpr (claims_tiles<MODE>()) {
        const int slot = it % GEMM_SCHED;
        ok = ok && mbar_wait(&sched_full[slot], (it / GEMM_SCHED) & 1, p.err);
        if (ok) {
          tile = sched[slot];
          rec = sched_rec[slot];
        }
      } else {
        tile = blockIdx.x + it * gridDim.x;
        if (tile >= n_tiles) tile = -1;
      }
      // the four epilogue warps leave together or not at all (they meet at
      // named barriers inside the tile); the claimed-tile slot is released
      // only after all of them have read it
      ok = named_bar_and(2, 128, ok);
      if constexpr (claims_tiles<MODE>()) {
        if (ok && etid == 0) mbar_arrive(&sched_empty[it % GEMM_SCHED]);
      }
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      if (tile < 0) break;
      GemmTile t;
      decode_tile<MODE>(p, tile, rec, n_gu, t);
      const int acc = it & 1;
      const uint32_t acc_par = (it >> 1) & 1;
      ok = mbar_wait(&tfull[acc], acc_par, p.err);
      ok = named_bar_and(2, 128, ok);
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * ACC_COLS * HALVES;

      if constexpr (MODE == GEMM_DENSE) {
        float* out = p.out_f32 + static_cast<size_t>(t.split) * p.T * p.M +
                     static_cast<size_t>(t.b_row) * p.M + t.a_row;
        if (p.use_tma_store && tile + static_cast<int>(gridDim.x) >= n_tiles) {
          // this CTA's last tile: every operand load has been consumed by the
          // MMAs this accumulator waited for, so the ring is free.  Stage the
          // tile as [token][128 features] fp32 (a warp writes 128 contiguous
          // bytes per token) and store it with TMA, 64 tokens per box.
          // Each 64-token box is stored as soon as it is staged, so the
          // stores overlap the staging of the next box.  Before the CTA exits
          // the stores must have read shared memory; kernel completion makes
          // their writes visible to the next launch.
          float* stage = reinterpret_cast<float*>(sA);
          for (int c0 = 0; c0 < t.n; c0 += 64) {
            float v[64];
            tmem_ld64(tbase + c0, v);
#pragma unroll
            for (int i = 0; i < 64; ++i) stage[(c0 + i) * GEMM_BM + row] = v[i];
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (etid == 0) {
              tma_store_3d(&p.out_map, stage + c0 * GEMM_BM, t.a_row, t.b_row + c0, t.split);
              bulk_commit_group();
            }
          }
          if (etid == 0) bulk_wait_read_all();
        } else
        for (int c0 = 0; c0 < t.n; c0 += 64) {
          float v[64];
          tmem_ld64(tbase + c0, v);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (c0 + 32 * h < t.n)
              store_rows_via_smem(xchg + h * 32 * GEMM_BM, v + 32 * h, row, etid,
                                  out + static_cast<size_t>(c0 + 32 * h) * p.M, p.M, min(32, t.n - c0 - 32 * h),
                                  p.M - t.a_row);
        }
      } else if constexpr (MODE == GEMM_MOE) {
        if (t.kind == KIND_GATEUP) {
          uint16_t* hout = t.shared ? p.hs_out : p.h_out;
          const int ld = t.shared ? p.Fs : p.F;
          const int col = t.blk * 64 + (row & 63);
          for (int c0 = 0; c0 < t.n; c0 += 32) {
            float v[32];
            tmem_ld32(tbase + c0, v);
            if (row < 64) {
#pragma unroll
              for (int i = 0; i < 32; ++i) xchg[row * 33 + i] = v[i];
            }
            named_bar_sync(1, 128);
            if (row >= 64) {
              const float* gv = xchg + (row - 64) * 33;
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int c = c0 + i;
                if (c < t.n) {
                  const float g = gv[i];
                  const float h = g / (1.f + __expf(-g)) * v[i];
                  hout[static_cast<size_t>(t.b_row + c) * ld + col] = f32_to_bf16(h);
                }
              }
            }
            named_bar_sync(1, 128);
          }
          // publish the hidden rows: every writer's stores are ordered before
          // one release increment of the chunk's counter
          __threadfence();
          fence_proxy_async_global();
          named_bar_sync(1, 128);
          if (etid == 0) red_release_gpu_add(p.chunk_done + t.chunk, 1);
        } else {
          const int r0 = (t.shared ? p.shared_row_base : 0) + t.b_row;
          float* out = p.out_f32 + static_cast<size_t>(r0) * p.out_ld + t.blk * GEMM_BM;
          for (int c0 = 0; c0 < t.n; c0 += 64) {
            float v[64];
            tmem_ld64(tbase + c0, v);
#pragma unroll
            for (int h = 0; h < 2; ++h)
              if (c0 + 32 * h < t.n)
                store_rows_via_smem(xchg + h * 32 * GEMM_BM, v + 32 * h, row, etid,
                                    out + static_cast<size_t>(c0 + 32 * h) * p.out_ld, p.out_ld,
                                    min(32, t.n - c0 - 32 * h), GEMM_BM);
          }
        }
      } else if (p.lse2 != nullptr) {  // GEMM_LMHEAD, probability mode
        for (int h = 0; h < t.halves; ++h) {
        const uint32_t th = tbase + h * ACC_COLS;
        const int y0 = t.a_row + h * GEMM_BM;
        // the previous store must have read the staging area
        if (etid == 0) bulk_wait_read_all();
        named_bar_sync(1, 128);
        const int tok = y0 + row;
        const float ref = tok < p.M ? p.lse2[tok] : 0.f;
        uint8_t* stg = reinterpret_cast<uint8_t*>(xchg);
        for (int c0 = 0; c0 < GEMM_BN; c0 += 32) {
          float v[32];
          tmem_ld32(th + c0, v);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(exp2f(fmaf(v[2 * i], p.logit_scale_log2, -ref)),
                                exp2f(fmaf(v[2 * i + 1], p.logit_scale_log2, -ref)));
          // two [128 rows][64 cols] boxes, 128-byte swizzle: 16-byte chunk ch of
          // row r sits at chunk (ch ^ (r & 7)) of the row
          const int box = c0 >> 6;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int ch = ((c0 & 63) >> 3) + q;
            *reinterpret_cast<uint4*>(stg + box * (GEMM_BM * 128) + row * 128 + ((ch ^ (row & 7)) << 4)) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (etid == 0) {
          tma_store_2d(&p.p_map, stg, t.b_row, y0);
          tma_store_2d(&p.p_map, stg + GEMM_BM * 128, t.b_row + 64, y0);
          bulk_commit_group();
        }
        }
      } else {  // GEMM_LMHEAD
        for (int h = 0; h < t.halves; ++h) {
        const uint32_t th = tbase + h * ACC_COLS;
        const int tok = t.a_row + h * GEMM_BM + row;
        float m1 = -INFINITY, m2 = -INFINITY, s = 0.f, s1 = 0.f;
        int idx = 0x7fffffff;
        for (int c0 = 0; c0 < GEMM_BN; c0 += 32) {
          float v[32];
          tmem_ld32(th + c0, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float x = v[i] * p.logit_scale_log2;
            if (x > m1) {
              m2 = m1;
              const float sc = exp2f(m1 - x);
              s = s * sc + 1.f;
              s1 = s1 * sc + x;
              m1 = x;
              idx = t.b_row + c0 + i;
            } else {
              m2 = fmaxf(m2, x);
              const float e = exp2f(x - m1);
              s += e;
              s1 = fmaf(e, x, s1);
            }
          }
        }
        if (tok < p.M) {
          p.lm_part[static_cast<size_t>(t.group) * p.M + tok] = make_float4(m1, __int_as_float(idx), m2, s);
          if (p.lm_s1) p.lm_s1[static_cast<size_t>(t.group) * p.M + tok] = s1;
        }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }

  // bulk stores have read shared memory before it is released (kernel
  // completion makes their writes visible to the next launch)
  if (MODE == GEMM_LMHEAD && p.lse2 != nullptr && threadIdx.x == 64) bulk_wait_read_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * ACC_COLS * HALVES);
  }
  if constexpr (claims_tiles<MODE>()) {
    // the last CTA out resets, for the next launch, the claim counter, the
    // per-expert row counts and the chunk flags (every CTA read the counts
    // and made its claims, and every flag wait ended, before its CTA counted
    // itself out)
    if (threadIdx.x == 0) {
      __threadfence();
      scan_tmp[0] = atomicAdd(p.work + 1, 1) == static_cast<int>(gridDim.x) - 1;
    }
    __syncthreads();
    if (scan_tmp[0]) {
      __threadfence();
      for (int e = threadIdx.x; e < p.n_groups_routed; e += blockDim.x) p.expert_rows[e] = 0;
      for (int c = threadIdx.x; c < tb_ch_off[tb.G]; c += blockDim.x) p.chunk_done[c] = 0;
      if (threadIdx.x == 0) {
        atomicExch(p.work, 0);
        atomicExch(p.work + 1, 0);
      }
    }
  }
}

}  // namespace dg
