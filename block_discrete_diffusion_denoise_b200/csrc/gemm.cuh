// Persistent, warp-specialised tcgen05 GEMM for sm_100a.
//
//   D[m, n] = sum_k A[m, k] * B[n, k]        (A, B bf16 K-major; D fp32 in TMEM)
//
// One CTA per SM.  Warp 0 (one lane) issues TMA loads into a 6-stage ring of
// shared-memory stages, warp 1 (one lane) issues tcgen05.mma into one of two
// TMEM accumulators (128 lanes x 128 fp32 columns each), warps 2..5 drain the
// other accumulator through the epilogue.  All waits are bounded.
//
// Four problem kinds share the pipeline (the tile decode and the epilogue
// differ):
//   DENSE   A = weight rows (output features), B = tokens; split-K partials
//           out[split][token][feature] fp32 (deterministic, no atomics).
//   GATEUP  grouped routed experts + the shared expert: A = 64 gate rows
//           stacked on the same 64 up rows, B = the expert's tokens; the
//           epilogue forms SiLU(gate) * up and stores bf16 hidden rows.
//   DOWN    grouped: A = 128 rows of the down projection, B = hidden rows;
//           fp32 output rows in permuted order.
//   LMHEAD  A = 128 tokens, B = 128 vocabulary rows of the tied embedding; the
//           epilogue keeps, per token, the running top-2 logits, the argmax
//           and the sum of exp, and writes one 16-byte partial per
//           (vocabulary tile, token) — the logits never reach memory.
#pragma once

#include "common.cuh"

namespace dg {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 64;
constexpr int GEMM_BN = 128;
constexpr int GEMM_STAGES = 6;
constexpr int GEMM_A_BYTES = GEMM_BM * GEMM_BK * 2;  // 16 KB
constexpr int GEMM_B_BYTES = GEMM_BN * GEMM_BK * 2;  // 16 KB
constexpr int GEMM_THREADS = 192;
constexpr int GEMM_TMEM_COLS = 2 * GEMM_BN;
constexpr int GEMM_XCHG_FLOATS = 64 * 33;            // gate values of one 32-column chunk
constexpr int GEMM_SMEM_BYTES = 1024 + GEMM_STAGES * (GEMM_A_BYTES + GEMM_B_BYTES) +
                                GEMM_XCHG_FLOATS * 4 + 256;

enum GemmMode : int { GEMM_DENSE = 0, GEMM_GATEUP = 1, GEMM_DOWN = 2, GEMM_LMHEAD = 3 };

struct GemmParams {
  CUtensorMap a_map[2];   // DENSE/DOWN/LMHEAD: [0]; GATEUP: [0] gate, [1] up   (routed)
  CUtensorMap as_map[2];  // shared expert A: GATEUP [0] gate, [1] up; DOWN [0]
  CUtensorMap b_map;      // DENSE: tokens; GATEUP: gathered rows; DOWN: hidden; LMHEAD: embed
  CUtensorMap bs_map;     // shared expert B: GATEUP: normed tokens; DOWN: shared hidden
  int b_box_rows;         // rows per B box (16 or 128)
  int M;                  // DENSE: output features; LMHEAD: tokens
  int T;                  // DENSE: tokens
  int k_steps;            // K / 64 (routed experts, dense, LM head)
  int k_steps_shared;     // K / 64 of the shared expert's down projection
  int splits;             // DENSE split-K
  int n_tiles_n;          // DENSE token tiles
  int bn;                 // DENSE token tile
  int n_mtiles;           // LMHEAD token tiles
  int tiles_static;       // DENSE / LMHEAD tile count
  const int* tile_count;  // GATEUP / DOWN: tile count (device)
  const int4* tiles;      // GATEUP / DOWN: {group, block, first row, rows}
  int n_groups_routed;    // group == n_groups_routed is the shared expert
  int a_rows_per_group;   // GATEUP: F; DOWN: d
  float* out_f32;         // DENSE partials [splits][T][M]; DOWN rows [.][out_ld]
  int out_ld;
  int shared_row_base;    // DOWN: output row of shared-expert token 0
  uint16_t* h_out;        // GATEUP routed hidden [rows][h_ld]
  uint16_t* hs_out;       // GATEUP shared hidden [tokens][hs_ld]
  int h_ld, hs_ld;
  float4* lm_part;        // LMHEAD partials [vocab tiles][M]
  float logit_scale_log2; // LMHEAD: log2(e) / temperature
  DevErr err;
};

struct GemmTile {
  const CUtensorMap* a0;
  const CUtensorMap* a1;  // second 64-row A box (GATEUP) or nullptr
  int a_row;
  const CUtensorMap* b;
  int b_row;
  int n;      // valid columns
  int nmma;   // MMA N (multiple of 16, <= 128)
  int k0, nk;
  int split, group, blk;
  bool a_stream;  // A is read once (evict-first)
};

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

template <int MODE>
__device__ __forceinline__ void decode_tile(const GemmParams& p, int tile, GemmTile& t) {
  if constexpr (MODE == GEMM_DENSE) {
    const int nt = tile % p.n_tiles_n;
    const int rest = tile / p.n_tiles_n;
    t.split = rest % p.splits;
    const int mt = rest / p.splits;
    t.a0 = &p.a_map[0];
    t.a1 = nullptr;
    t.a_row = mt * GEMM_BM;
    t.b = &p.b_map;
    t.b_row = nt * p.bn;
    t.n = min(p.bn, p.T - t.b_row);
    t.nmma = round16(t.n);
    t.k0 = (t.split * p.k_steps) / p.splits;
    t.nk = ((t.split + 1) * p.k_steps) / p.splits - t.k0;
    t.group = 0;
    t.blk = mt;
    t.a_stream = p.n_tiles_n == 1;
  } else if constexpr (MODE == GEMM_LMHEAD) {
    const int vt = tile / p.n_mtiles;
    const int mt = tile % p.n_mtiles;
    t.a0 = &p.a_map[0];
    t.a1 = nullptr;
    t.a_row = mt * GEMM_BM;
    t.b = &p.b_map;
    t.b_row = vt * GEMM_BN;
    t.n = GEMM_BN;
    t.nmma = GEMM_BN;
    t.k0 = 0;
    t.nk = p.k_steps;
    t.split = 0;
    t.group = vt;
    t.blk = mt;
    t.a_stream = false;
  } else {
    const int4 e = p.tiles[tile];
    const bool shared = e.x == p.n_groups_routed;
    t.group = e.x;
    t.blk = e.y;
    t.b_row = e.z;
    t.n = e.w;
    t.nmma = round16(e.w);
    t.k0 = 0;
    t.split = 0;
    t.a_stream = !shared;
    if constexpr (MODE == GEMM_GATEUP) {
      t.a0 = shared ? &p.as_map[0] : &p.a_map[0];
      t.a1 = shared ? &p.as_map[1] : &p.a_map[1];
      t.a_row = (shared ? 0 : e.x * p.a_rows_per_group) + e.y * 64;
      t.b = shared ? &p.bs_map : &p.b_map;
      t.nk = p.k_steps;
    } else {
      t.a0 = shared ? &p.as_map[0] : &p.a_map[0];
      t.a1 = nullptr;
      t.a_row = (shared ? 0 : e.x * p.a_rows_per_group) + e.y * GEMM_BM;
      t.b = shared ? &p.bs_map : &p.b_map;
      t.nk = shared ? p.k_steps_shared : p.k_steps;
    }
  }
}

template <int MODE>
__device__ __forceinline__ int tile_total(const GemmParams& p) {
  if constexpr (MODE == GEMM_GATEUP || MODE == GEMM_DOWN) return *p.tile_count;
  return p.tiles_static;
}

// -----------------------------------------------------------------------------
// epilogues: thread owns TMEM lane (row) `row` of the tile; v = 32 columns
// -----------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(GEMM_THREADS, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + GEMM_STAGES * GEMM_A_BYTES;
  float* xchg = reinterpret_cast<float*>(sB + GEMM_STAGES * GEMM_B_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(xchg + GEMM_XCHG_FLOATS);
  uint64_t* empty = full + GEMM_STAGES;
  uint64_t* tfull = empty + GEMM_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tiles = tile_total<MODE>(p);

  if (threadIdx.x == 0) {
    for (int s = 0; s < GEMM_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, GEMM_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&p.a_map[0]);
      tma_prefetch_desc(&p.b_map);
      const uint64_t pol_first = policy_evict_first();
      const uint64_t pol_last = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_par = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort_flag; tile += gridDim.x) {
        GemmTile t;
        decode_tile<MODE>(p, tile, t);
        const uint32_t bytes = GEMM_A_BYTES + t.nmma * GEMM_BK * 2;
        const uint64_t pol_a = (MODE == GEMM_LMHEAD) ? pol_last : (t.a_stream ? pol_first : pol_last);
        const uint64_t pol_b = (MODE == GEMM_LMHEAD) ? pol_last : pol_last;
        for (int k = 0; k < t.nk; ++k) {
          if (!mbar_wait(&empty[stage], phase ^ 1, p.err)) {
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], bytes);
          uint8_t* a = sA + stage * GEMM_A_BYTES;
          uint8_t* b = sB + stage * GEMM_B_BYTES;
          const int kx = (t.k0 + k) * GEMM_BK;
          if (t.a1 != nullptr) {
            tma_load_2d(a, t.a0, &full[stage], kx, t.a_row, pol_a);
            tma_load_2d(a + GEMM_A_BYTES / 2, t.a1, &full[stage], kx, t.a_row, pol_a);
          } else {
            tma_load_2d(a, t.a0, &full[stage], kx, t.a_row, pol_a);
          }
          for (int r = 0; r < t.nmma; r += p.b_box_rows)
            tma_load_2d(b + r * (GEMM_BK * 2), t.b, &full[stage], kx, t.b_row + r, pol_b);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == GEMM_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // every copy this thread issued has landed before the CTA may exit
      for (int s = 0; s < GEMM_STAGES; ++s)
        if ((issued >> s) & 1) mbar_wait(&full[s], (issued_par >> s) & 1, p.err);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool aborted = false;
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
        if (*abort_flag) {
          aborted = true;
          break;
        }
        GemmTile t;
        decode_tile<MODE>(p, tile, t);
        const int acc = it & 1;
        const uint32_t acc_par = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_par ^ 1, p.err)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * GEMM_BN;
        const uint32_t idesc = umma_idesc_bf16(GEMM_BM, t.nmma);
        for (int k = 0; k < t.nk; ++k) {
          if (!mbar_wait(&full[stage], phase, p.err)) {
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint64_t ad = umma_desc_sw128(smem_u32(sA + stage * GEMM_A_BYTES));
          const uint64_t bd = umma_desc_sw128(smem_u32(sB + stage * GEMM_B_BYTES));
#pragma unroll
          for (int kk = 0; kk < GEMM_BK / 16; ++kk)
            umma_bf16(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (k | kk) != 0);
          umma_commit(&empty[stage]);
          if (++stage == GEMM_STAGES) {
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
    // ------------------------------ epilogue ----------------------------------
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;       // tile row owned by this thread
    int it = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      GemmTile t;
      decode_tile<MODE>(p, tile, t);
      const int acc = it & 1;
      const uint32_t acc_par = (it >> 1) & 1;
      bool ok = (*abort_flag == 0) && mbar_wait(&tfull[acc], acc_par, p.err);
      // the four epilogue warps leave together or not at all (they meet at
      // named barriers inside the tile)
      ok = named_bar_and(2, 128, ok);
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * GEMM_BN;

      if constexpr (MODE == GEMM_DENSE) {
        const int m = t.a_row + row;
        float* out = p.out_f32 + static_cast<size_t>(t.split) * p.T * p.M;
        for (int c0 = 0; c0 < t.n; c0 += 32) {
          float v[32];
          tmem_ld32(tbase + c0, v);
          if (m < p.M) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int c = c0 + i;
              if (c < t.n) out[static_cast<size_t>(t.b_row + c) * p.M + m] = v[i];
            }
          }
        }
      } else if constexpr (MODE == GEMM_GATEUP) {
        const bool shared = t.group == p.n_groups_routed;
        uint16_t* hout = shared ? p.hs_out : p.h_out;
        const int ld = shared ? p.hs_ld : p.h_ld;
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
      } else if constexpr (MODE == GEMM_DOWN) {
        const bool shared = t.group == p.n_groups_routed;
        const int m = t.blk * GEMM_BM + row;
        const int r0 = (shared ? p.shared_row_base : 0) + t.b_row;
        for (int c0 = 0; c0 < t.n; c0 += 32) {
          float v[32];
          tmem_ld32(tbase + c0, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int c = c0 + i;
            if (c < t.n) p.out_f32[static_cast<size_t>(r0 + c) * p.out_ld + m] = v[i];
          }
        }
      } else {  // GEMM_LMHEAD
        const int tok = t.a_row + row;
        float m1 = -INFINITY, m2 = -INFINITY, s = 0.f;
        int idx = 0x7fffffff;
        for (int c0 = 0; c0 < GEMM_BN; c0 += 32) {
          float v[32];
          tmem_ld32(tbase + c0, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float x = v[i] * p.logit_scale_log2;
            if (x > m1) {
              m2 = m1;
              s = s * exp2f(m1 - x) + 1.f;
              m1 = x;
              idx = t.b_row + c0 + i;
            } else {
              m2 = fmaxf(m2, x);
              s += exp2f(x - m1);
            }
          }
        }
        if (tok < p.M)
          p.lm_part[static_cast<size_t>(t.group) * p.M + tok] = make_float4(m1, __int_as_float(idx), m2, s);
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, GEMM_TMEM_COLS);
  }
}

}  // namespace dg
