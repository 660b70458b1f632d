// Grouped-query attention on tcgen05 tensor cores (sm_100a), two masks:
//   causal:        query i (position pos0 + i) sees keys [0, pos0 + i]
//   bidirectional: every query sees keys [0, pos0 + n)   (cache + whole canvas)
// (codemajin.net "DiffusionGemma architecture", section 3.2: the causal encoder
// fills the KV cache, the bidirectional decoder reads it while updating the
// whole canvas; aiboss88.com "hybrid attention architecture" names both modes.)
//
// One CTA = (sequence, kv head, 256 packed query rows, key chunk).  The G
// query heads of a GQA group are packed as consecutive rows (row = i*G + h)
// so each K/V block feeds all of them; the 256 rows are two 128-row query
// tiles, each pulled by one 4-D TMA box out of the [token][head][D] query
// layout, and every K/V block is read once for both.  The keys are split
// into chunks so the grid fills the SMs; with one chunk a CTA writes its
// normalised rows, with several it writes its raw rows and row statistics to
// a partial buffer and attn_merge_kernel combines them.
//
// Warp 0 issues TMA loads (lane 0: both Q tiles once, then 64-key K blocks;
// lane 1: V blocks; 2-deep rings).  Warp 1 issues tcgen05.mma: S_q = Q_q K^T into tile q's TMEM
// buffer (128 x 64 fp32) and O_q += P_q V into tile q's TMEM accumulator
// (128 x D fp32; V used as an MN-major operand).  Warps 2..5 and 6..9 are the
// softmax warpgroups of tiles 0 and 1, one query row per thread, so every row
// statistic is thread-local.  While one warpgroup turns its S into P the
// tensor core works on the other tile.
//
// Single pass with online softmax: P = 2^(s * scale - m_ref), where m_ref is a
// per-row reference maximum.  It is raised only when a block's maximum
// exceeds it by more than RESCALE_LOG2 (then O and the row sum are scaled by
// 2^(old - new) in TMEM), so P stays below 2^RESCALE_LOG2 and rescaling is
// rare after the first block.
#pragma once

#include "common.cuh"

namespace dg {

constexpr int ATC_BQ = 128;        // packed query rows per tile (MMA M)
constexpr int ATC_NQ = 2;          // query tiles per CTA
constexpr int ATC_ROWS = ATC_BQ * ATC_NQ;
constexpr int ATC_BK = 64;         // keys per block (MMA N of Q K^T, K of P V)
constexpr int ATC_KSTAGES = 2;
constexpr int ATC_VSTAGES = 2;
constexpr int ATC_THREADS = 320;   // producer warp, MMA warp, two softmax warpgroups
constexpr int ATC_MAX_CHUNKS = 10; // key chunks per query block (combined by attn_merge_kernel)
constexpr float ATC_RESCALE_LOG2 = 8.f;

struct AttnTcParams {
  CUtensorMap q_map;   // 4-D (D, G, Hkv, tokens) over q [token][Hq][D]; box (64, G, 1, 128/G)
  CUtensorMap k_map;   // 2-D (D, B*Hkv*S_max) over this layer's K cache; box (64, 64)
  CUtensorMap v_map;   // same over V
  uint16_t* o;         // [token][Hq][D]
  float* part;         // several key chunks: [unit][chunk][D/4][256 rows] float4 raw rows (unit = y * qblocks + x)
  float2* part_ml;     // [unit][chunk][256 rows] (max, sum) of those rows
  int n, B, Hq, Hkv, S_max, pos0, causal, chunk_len, n_chunks;
  float scale_log2;    // log2(e) / sqrt(D)
  DevErr err;
};

template <int D>
struct AtcCfg {
  static constexpr int DK = (D + 63) / 64;             // 64-column boxes along the head dimension
  static constexpr int Q_BYTES = DK * ATC_BQ * 128;    // one query tile
  static constexpr int KV_BYTES = DK * ATC_BK * 128;
  static constexpr int P_BYTES = ATC_BQ * ATC_BK * 2;  // one tile's P
  static constexpr int REGION = ATC_NQ * Q_BYTES + (ATC_KSTAGES + ATC_VSTAGES) * KV_BYTES + ATC_NQ * P_BYTES;
  static constexpr int S_COL = 0;                      // TMEM: S_q at q * 64, O_q at 128 + q * D
  static constexpr int O_COL = ATC_NQ * ATC_BK;
  static constexpr int TMEM_COLS = O_COL + ATC_NQ * D <= 256 ? 256 : 512;
  static constexpr int TAIL = 512;                     // barriers, flags
  static constexpr int SMEM = 1024 + REGION + TAIL;
  static_assert(O_COL + ATC_NQ * D <= 512, "S and O accumulators must fit TMEM");
  static_assert(D % 16 == 0 && D <= 256, "head_dim must be a multiple of 16, at most 256");
};

template <int D>
__global__ void __launch_bounds__(ATC_THREADS, 1) attn_tc_kernel(const __grid_constant__ AttnTcParams p) {
  DG_TIMELINE_SCOPE(TLK_ATTENTION);
  using C = AtcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sQ = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = sQ + ATC_NQ * C::Q_BYTES;
  uint8_t* sV = sK + ATC_KSTAGES * C::KV_BYTES;
  uint8_t* sP = sV + ATC_VSTAGES * C::KV_BYTES;
  uint8_t* tail = sQ + C::REGION;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tail);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + ATC_KSTAGES;
  uint64_t* v_full = k_empty + ATC_KSTAGES;
  uint64_t* v_empty = v_full + ATC_VSTAGES;
  uint64_t* s_full = v_empty + ATC_VSTAGES;   // [NQ] MMA -> warpgroup q: S_q of the next block ready
  uint64_t* s_free = s_full + ATC_NQ;         // [NQ] warpgroup q -> MMA: S_q read into registers
  uint64_t* p_full = s_free + ATC_NQ;         // [NQ] warpgroup q -> MMA: P_q written
  uint64_t* o_done = p_full + ATC_NQ;         // [NQ] MMA -> warpgroup q: O_q += P_q V complete
  uint64_t* drain = o_done + ATC_NQ;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tail + 256);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tail + 260);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.Hq / p.Hkv;
  const int b = blockIdx.y / p.Hkv, kvh = blockIdx.y % p.Hkv;
  const int rows_total = p.n * G;
  const int row_base = blockIdx.x * ATC_ROWS;
  const int nq = rows_total - row_base > ATC_BQ ? 2 : 1;   // query tiles holding live rows
  int kend_cta;
  if (p.causal) {
    const int i_last = min((row_base + nq * ATC_BQ - 1) / G, p.n - 1);
    kend_cta = p.pos0 + i_last + 1;
  } else {
    kend_cta = p.pos0 + p.n;
  }
  const int kbeg = blockIdx.z * p.chunk_len;
  const int kend = min(kbeg + p.chunk_len, kend_cta);
  const int nb = kend > kbeg ? (kend - kbeg + ATC_BK - 1) / ATC_BK : 0;
  const int kv_row0 = (b * p.Hkv + kvh) * p.S_max + kbeg;

  if (threadIdx.x == 0) {
    // the descriptors are fetched while the CTA sets up
    tma_prefetch_desc(&p.q_map);
    tma_prefetch_desc(&p.k_map);
    tma_prefetch_desc(&p.v_map);
    mbar_init(q_full, 1);
    for (int s = 0; s < ATC_KSTAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < ATC_VSTAGES; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int q = 0; q < ATC_NQ; ++q) {
      mbar_init(&s_full[q], 1);
      mbar_init(&s_free[q], ATC_BQ);
      mbar_init(&p_full[q], ATC_BQ);
      mbar_init(&o_done[q], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // softmax state of this thread's row (warps 2..9)
  const int wg = (warp - 2) >> 2;                // softmax warpgroup = query tile
  const int quarter = warp & 3;                  // TMEM lanes this warp may access
  const int rloc = quarter * 32 + lane;          // row of the tile = TMEM lane
  const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
  const int r = row_base + wg * ATC_BQ + rloc;
  const bool live = r < rows_total;
  float mref = -INFINITY, lsum = 0.f;
  bool ok = true;

  if (warp == 0) {
    // ------------------------ TMA producers: lane 0 K, lane 1 V ------------------------
    // Separate lanes, so a K block is requested as soon as its ring slot is
    // free, whatever the V ring is waiting for (and the other way round).
    if (lane < 2 && nb > 0) {
      const bool kl = lane == 0;
      const CUtensorMap* map = kl ? &p.k_map : &p.v_map;
      uint64_t* full = kl ? k_full : v_full;
      uint64_t* empty = kl ? k_empty : v_empty;
      uint8_t* ring = kl ? sK : sV;
      constexpr int NS = ATC_KSTAGES;  // both rings have the same depth
      static_assert(ATC_KSTAGES == ATC_VSTAGES, "K and V rings are walked by the same loop");
      tma_prefetch_desc(map);
      const uint64_t pol = policy_evict_last();  // K/V blocks are shared by the head's query blocks
      uint32_t issued = 0, par = 0;
      if (kl) {
        tma_prefetch_desc(&p.q_map);
        mbar_arrive_expect_tx(q_full, nq * C::Q_BYTES);
        for (int q = 0; q < nq; ++q)
          for (int db = 0; db < C::DK; ++db)
            tma_load_4d(sQ + q * C::Q_BYTES + db * ATC_BQ * 128, &p.q_map, q_full, db * 64, 0, kvh,
                        b * p.n + (row_base + q * ATC_BQ) / G, pol);
      }
      for (int j = 0; j < nb && !*abort_flag; ++j) {
        const int s = j % NS;
        const uint32_t ph = (j / NS) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.err)) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[s], C::KV_BYTES);
        for (int db = 0; db < C::DK; ++db)
          tma_load_2d(ring + s * C::KV_BYTES + db * ATC_BK * 128, map, &full[s], db * 64, kv_row0 + j * ATC_BK,
                      pol);
        issued |= 1u << s;
        par = (par & ~(1u << s)) | (ph << s);
      }
      // every copy issued here has landed before its buffer is reused or the CTA exits
      if (kl) mbar_wait(q_full, 0, p.err);
      for (int s = 0; s < NS; ++s)
        if ((issued >> s) & 1) mbar_wait(&full[s], (par >> s) & 1, p.err);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    // An event loop: each pass issues every S = Q K^T and every O += P V
    // whose inputs are ready (non-blocking tests), scores first.  A score
    // tile waits only for its K block and for its warpgroup to have read the
    // previous scores; a P V product only for its V block and its P.
    if (lane == 0 && nb > 0) {
      constexpr uint32_t IDESC_S = umma_idesc_bf16(ATC_BQ, ATC_BK);             // Q, K both K-major
      constexpr uint32_t IDESC_PV = umma_idesc_bf16(ATC_BQ, D) | (1u << 16);    // V is MN-major
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV), p_addr = smem_u32(sP);
      bool mok = mbar_wait(q_full, 0, p.err);
      tc_fence_after();
      int ns[ATC_NQ] = {0, 0}, np[ATC_NQ] = {0, 0};
      uint64_t t_idle = globaltimer_ns();
      while (mok && (np[0] < nb || (nq == 2 && np[1] < nb))) {
        bool prog = false;
        for (int q = 0; q < nq; ++q) {
          const int j = ns[q];
          if (j < nb && (j == 0 || mbar_try_wait(&s_free[q], (j - 1) & 1)) &&
              mbar_try_wait(&k_full[j % ATC_KSTAGES], (j / ATC_KSTAGES) & 1)) {
            tc_fence_after();
            const uint32_t kb = k_addr + (j % ATC_KSTAGES) * C::KV_BYTES, qb = q_addr + q * C::Q_BYTES;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t a_at = qb + (kk >> 2) * (ATC_BQ * 128) + (kk & 3) * 32;
              const uint32_t b_at = kb + (kk >> 2) * (ATC_BK * 128) + (kk & 3) * 32;
              umma_bf16(tmem_base + C::S_COL + q * ATC_BK, umma_desc_sw128(a_at), umma_desc_sw128(b_at), IDESC_S,
                        kk > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[q]);
            ns[q] = j + 1;
            // the K slot is released once every live tile has read block j
            if (ns[0] > j && (nq < 2 || ns[1] > j)) umma_commit(&k_empty[j % ATC_KSTAGES]);
            prog = true;
          }
        }
        for (int q = 0; q < nq; ++q) {
          const int j = np[q];
          if (j < ns[q] && mbar_try_wait(&v_full[j % ATC_VSTAGES], (j / ATC_VSTAGES) & 1) &&
              mbar_try_wait(&p_full[q], j & 1)) {
            tc_fence_after();
            const uint32_t vb = v_addr + (j % ATC_VSTAGES) * C::KV_BYTES, pb = p_addr + q * C::P_BYTES;
#pragma unroll
            for (int kk = 0; kk < ATC_BK / 16; ++kk)
              umma_bf16(tmem_base + C::O_COL + q * D, umma_desc_sw128(pb + kk * 32),
                        umma_desc_sw128_mn(vb + kk * 2048, ATC_BK * 128), IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
            umma_commit(&o_done[q]);
            np[q] = j + 1;
            if (np[0] > j && (nq < 2 || np[1] > j)) umma_commit(&v_empty[j % ATC_VSTAGES]);
            prog = true;
          }
        }
        if (prog) {
          t_idle = globaltimer_ns();
        } else if (*abort_flag) {
          mok = false;
        } else if (globaltimer_ns() - t_idle > p.err.limit_ns) {
          raise_error(p.err, ERR_TIMEOUT);
          mok = false;
        }
      }
      if (!mok) *abort_flag = 1;
      // every MMA issued has completed before TMEM or its operands are reused
      umma_commit(drain);
      mbar_wait(drain, 0, p.err);
    }
  } else if (wg < nq && nb > 0) {
    // ----------------------- softmax warpgroup of tile wg -----------------------
    const int i = live ? r / G : 0;
    // keys of this chunk the row sees: [0, lim) relative to kbeg
    const int lim = (live ? min(p.causal ? p.pos0 + i + 1 : p.pos0 + p.n, kend) : 0) - kbeg;
    const uint32_t s_col = t_row + C::S_COL + wg * ATC_BK;
    const uint32_t o_col = t_row + C::O_COL + wg * D;
    uint8_t* pdst = sP + wg * C::P_BYTES + rloc * 128;
    float s[64];
    for (int j = 0; j < nb && ok; ++j) {
      // warp-uniform decision: tcgen05.ld below is a warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[wg], j & 1, p.err) && !*abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_ld64(s_col, s);
      tc_fence_before();
      mbar_arrive(&s_free[wg]);
      const int lj = lim - j * ATC_BK;
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (lj >= ATC_BK) {
#pragma unroll
        for (int c = 0; c < ATC_BK; ++c) mx[c & 3] = fmaxf(mx[c & 3], s[c]);
      } else {
#pragma unroll
        for (int c = 0; c < ATC_BK; ++c)
          if (c < lj) mx[c & 3] = fmaxf(mx[c & 3], s[c]);
      }
      // scale > 0, so the maximum of the scaled scores is the scaled maximum
      const float mblk = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
      const bool resc = mblk > mref + ATC_RESCALE_LOG2;          // false while nothing is visible
      const float factor = resc ? ex2_approx(mref - mblk) : 1.f;  // 0 when mref = -inf
      if (resc) mref = mblk;
      lsum *= factor;
      float l = 0.f;
      uint32_t pk[ATC_BK / 2];
#pragma unroll
      for (int c = 0; c < ATC_BK / 2; ++c) {
        const float p0 = (2 * c < lj) ? ex2_approx(fmaf(s[2 * c], p.scale_log2, -mref)) : 0.f;
        const float p1 = (2 * c + 1 < lj) ? ex2_approx(fmaf(s[2 * c + 1], p.scale_log2, -mref)) : 0.f;
        l += p0 + p1;
        pk[c] = pack_bf16x2(p0, p1);
      }
      lsum += l;
      if (j > 0) {
        // O_q += P_q(j-1) V_{j-1} has completed: O_q is stable and P_q's buffer free
        if (!__all_sync(0xffffffffu, mbar_wait(&o_done[wg], (j - 1) & 1, p.err))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 16) {
            float v[16];
            tmem_ld16(o_col + c0, v);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] *= factor;
            tmem_st16(o_col + c0, v);
          }
          tmem_st_wait();
        }
      }
      // row rloc of a K-major 128-byte-swizzled tile: 16-byte chunk c lands at c ^ (row & 7)
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        *reinterpret_cast<uint4*>(pdst + ((ch ^ (rloc & 7)) << 4)) =
            make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[wg]);
    }
    if (ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(&o_done[wg], (nb - 1) & 1, p.err) && !*abort_flag);
      tc_fence_after();
    }
    if (!ok) *abort_flag = 1;
  }

  // ---------- one chunk: the rows; several: the partials for the merge ----------
  const int nc = p.n_chunks;
  if (warp >= 2) {
    named_bar_sync(1, 256);  // both tiles' MMAs are complete
    const bool have = wg < nq && nb > 0 && ok;
    if (!have) {
      mref = -INFINITY;
      lsum = 0.f;
    }
  }
  const bool have_o = warp >= 2 && wg < nq && nb > 0 && __all_sync(0xffffffffu, ok);  // warp-uniform
  const int row = (warp >= 2) ? wg * ATC_BQ + rloc : 0;
  if (nc == 1) {
    // one chunk: normalise and store this thread's row directly
    if (warp >= 2) {
      const int rg = row_base + row;
      const float w = lsum > 0.f ? 1.f / lsum : 0.f;
      const size_t rid = (static_cast<size_t>(b) * p.n + rg / G) * p.Hq + kvh * G + rg % G;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 16) {
        float v[16];
        if (have_o) {
          tmem_ld16(t_row + C::O_COL + wg * D + c0, v);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = 0.f;
        }
        if (rg < rows_total) {
          uint4* dst = reinterpret_cast<uint4*>(p.o + rid * D + c0);
          dst[0] = make_uint4(pack_bf16x2(v[0] * w, v[1] * w), pack_bf16x2(v[2] * w, v[3] * w),
                              pack_bf16x2(v[4] * w, v[5] * w), pack_bf16x2(v[6] * w, v[7] * w));
          dst[1] = make_uint4(pack_bf16x2(v[8] * w, v[9] * w), pack_bf16x2(v[10] * w, v[11] * w),
                              pack_bf16x2(v[12] * w, v[13] * w), pack_bf16x2(v[14] * w, v[15] * w));
        }
      }
    }
  } else if (warp >= 2) {
    // several key chunks: this chunk's raw rows and their (max, sum) go to its
    // slot of the partial buffer, [unit][chunk][D/4][256 rows] float4 (a
    // warp's store covers 32 consecutive rows, 512 contiguous bytes);
    // attn_merge_kernel combines the chunks
    constexpr int D4 = D / 4;
    const size_t slot = (static_cast<size_t>(blockIdx.y) * gridDim.x + blockIdx.x) * nc + blockIdx.z;
    float4* dst = reinterpret_cast<float4*>(p.part) + slot * D4 * ATC_ROWS + row;
    p.part_ml[slot * ATC_ROWS + row] = make_float2(have_o ? mref : -INFINITY, have_o ? lsum : 0.f);
    auto put16 = [&](int c0, const float* v) {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        dst[static_cast<size_t>(c0 / 4 + e) * ATC_ROWS] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    };
    int c0 = 0;
#pragma unroll 1
    for (; c0 + 32 <= D; c0 += 32) {
      float v[32];
      if (have_o) {
        tmem_ld32(t_row + C::O_COL + wg * D + c0, v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.f;
      }
      put16(c0, v);
      put16(c0 + 16, v + 16);
    }
    if (c0 < D) {  // D is a multiple of 16
      float v[16];
      if (have_o) {
        tmem_ld16(t_row + C::O_COL + wg * D + c0, v);
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = 0.f;
      }
      put16(c0, v);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// Merge of the key chunks of attn_tc_kernel (several chunks):
//   o = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c,  M = max_c m_c,
// summed in chunk order.  One thread per (unit, row, 4-column group):
// consecutive threads take consecutive rows of one group, so the partial and
// row-statistic loads are coalesced, and every load a thread needs (nc
// partials, nc statistics) is issued before the first is used: one memory
// round trip, no shared memory.  grid = (units, 256 * D/4 / 256), 256 threads.
template <int D>
__global__ void __launch_bounds__(256, 3) attn_merge_kernel(const float4* __restrict__ part,
                                                         const float2* __restrict__ part_ml, int nc, int qblocks,
                                                         int n, int Hq, int Hkv, uint16_t* __restrict__ o) {
  DG_TIMELINE_SCOPE(TLK_ATTN_MERGE);
  constexpr int D4 = D / 4;
  const int unit = blockIdx.x;  // = blockIdx.y * qblocks + blockIdx.x of the attention launch
  const int it = blockIdx.y * blockDim.x + threadIdx.x;
  if (it >= ATC_ROWS * D4) return;
  const int r = it % ATC_ROWS, c4 = it / ATC_ROWS;
  const int qb = unit % qblocks, bk = unit / qblocks;
  const int b = bk / Hkv, kvh = bk % Hkv;
  const int G = Hq / Hkv, rows_total = n * G;
  const size_t slot0 = static_cast<size_t>(unit) * nc;
  const float4* src = part + slot0 * D4 * ATC_ROWS + static_cast<size_t>(c4) * ATC_ROWS + r;
  float2 ml[ATC_MAX_CHUNKS];
  float4 v[ATC_MAX_CHUNKS];
#pragma unroll
  for (int q = 0; q < ATC_MAX_CHUNKS; ++q)
    if (q < nc) {
      ml[q] = part_ml[(slot0 + q) * ATC_ROWS + r];
      v[q] = src[static_cast<size_t>(q) * D4 * ATC_ROWS];
    }
  float M = -INFINITY;
#pragma unroll
  for (int q = 0; q < ATC_MAX_CHUNKS; ++q)
    if (q < nc) M = fmaxf(M, ml[q].x);
  const float Mref = M == -INFINITY ? 0.f : M;
  float den = 0.f;
#pragma unroll
  for (int q = 0; q < ATC_MAX_CHUNKS; ++q)
    if (q < nc && ml[q].x != -INFINITY) den += ml[q].y * ex2_approx(ml[q].x - Mref);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int q = 0; q < ATC_MAX_CHUNKS; ++q)
    if (q < nc) {
      const float wq = (den > 0.f && ml[q].x != -INFINITY) ? ex2_approx(ml[q].x - Mref) / den : 0.f;
      acc.x = fmaf(v[q].x, wq, acc.x);
      acc.y = fmaf(v[q].y, wq, acc.y);
      acc.z = fmaf(v[q].z, wq, acc.z);
      acc.w = fmaf(v[q].w, wq, acc.w);
    }
  const int rg = qb * ATC_ROWS + r;
  if (rg >= rows_total) return;
  const size_t rid = (static_cast<size_t>(b) * n + rg / G) * Hq + kvh * G + rg % G;
  *reinterpret_cast<uint2*>(o + rid * D + 4 * c4) = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
}

}  // namespace dg
