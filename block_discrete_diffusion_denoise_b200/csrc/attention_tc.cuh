// Grouped-query attention on tcgen05 tensor cores (sm_100a), two masks:
//   causal:        query i (position pos0 + i) sees keys [0, pos0 + i]
//   bidirectional: every query sees keys [0, pos0 + n)   (cache + whole canvas)
// (codemajin.net "DiffusionGemma architecture", section 3.2: the causal encoder
// fills the KV cache, the bidirectional decoder reads it while updating the
// whole canvas; aiboss88.com "hybrid attention architecture" names both modes.)
//
// One CTA = (sequence, kv head, 128 packed query rows, key chunk).  The G
// query heads of a GQA group are packed as consecutive rows (row = i*G + h)
// so each K/V block feeds all of them; a 4-D TMA box pulls exactly those rows
// out of the [token][head][D] query layout.  The key chunks of one query block
// form a thread-block cluster and are merged through distributed shared memory.
//
// Warp 0 issues TMA loads (Q once; 64-key K blocks into a 3-deep ring; V blocks
// into a 2-deep ring).  Warp 1 issues tcgen05.mma: S = Q K^T into one of two
// TMEM buffers (128 x 64 fp32), and O += P V into TMEM (128 x D fp32; V used as
// an MN-major operand).  Warps 2..5 and 6..9 are two softmax warpgroups; each
// owns one S buffer (even / odd S tiles) and one query row per thread.
//
// Two passes over the key blocks: pass 1 only finds each row's maximum score;
// pass 2 recomputes S, forms P = 2^(s*scale - max) (bf16, written to shared
// memory in the swizzled K-major operand layout) and the row sums.  With the
// final maximum known up front, O never needs rescaling inside TMEM.
#pragma once

#include "common.cuh"

namespace dg {

constexpr int ATC_BQ = 128;        // packed query rows per CTA (MMA M)
constexpr int ATC_BK = 64;         // keys per block (MMA N of Q K^T, K of P V)
constexpr int ATC_KSTAGES = 3;
constexpr int ATC_VSTAGES = 2;
constexpr int ATC_THREADS = 320;   // producer warp, MMA warp, two softmax warpgroups
constexpr int ATC_MAX_CHUNKS = 8;  // key chunks = cluster size (portable limit)

struct AttnTcParams {
  CUtensorMap q_map;   // 4-D (D, G, Hkv, tokens) over q [token][Hq][D]; box (64, G, 1, 128/G)
  CUtensorMap k_map;   // 2-D (D, B*Hkv*S_max) over this layer's K cache; box (64, 64)
  CUtensorMap v_map;   // same over V
  uint16_t* o;         // [token][Hq][D]
  int n, B, Hq, Hkv, S_max, pos0, causal, chunk_len, n_chunks;
  float scale_log2;    // log2(e) / sqrt(D)
  DevErr err;
};

template <int D>
struct AtcCfg {
  static constexpr int DK = (D + 63) / 64;             // 64-column boxes along the head dimension
  static constexpr int Q_BYTES = DK * ATC_BQ * 128;
  static constexpr int KV_BYTES = DK * ATC_BK * 128;
  static constexpr int P_BYTES = ATC_BQ * ATC_BK * 2;
  static constexpr int O_COL = 128;                    // TMEM: S buffers in columns [0, 128), O after them
  static constexpr int TMEM_COLS = O_COL + D <= 256 ? 256 : 512;
  static constexpr int OS_LD = D + 4;                  // fp32 row stride of the merged-O staging tile
  static constexpr int TAIL = 4096;                    // barriers, flags, row statistics
  static constexpr int SMEM = 1024 + Q_BYTES + (ATC_KSTAGES + ATC_VSTAGES) * KV_BYTES + 2 * P_BYTES + TAIL;
  static_assert(ATC_BQ * OS_LD * 4 <= (ATC_KSTAGES + ATC_VSTAGES) * KV_BYTES, "O staging must fit the K/V ring");
  static_assert(D % 16 == 0 && D <= 256, "head_dim must be a multiple of 16, at most 256");
};

template <int D>
__global__ void __launch_bounds__(ATC_THREADS, 1) attn_tc_kernel(const __grid_constant__ AttnTcParams p) {
  using C = AtcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sQ = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = sQ + C::Q_BYTES;
  uint8_t* sV = sK + ATC_KSTAGES * C::KV_BYTES;
  uint8_t* sP = sV + ATC_VSTAGES * C::KV_BYTES;
  uint8_t* tail = sP + 2 * C::P_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tail);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + ATC_KSTAGES;
  uint64_t* v_full = k_empty + ATC_KSTAGES;
  uint64_t* v_empty = v_full + ATC_VSTAGES;
  uint64_t* s_full = v_empty + ATC_VSTAGES;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* p_empty = p_full + 2;
  uint64_t* o_full = p_empty + 2;
  uint64_t* drain = o_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tail + 256);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tail + 260);
  float* red_m = reinterpret_cast<float*>(tail + 512);           // [2][128] per-warpgroup row maxima
  float* red_l = red_m + 2 * ATC_BQ;                             // [2][128] per-warpgroup row sums
  float2* ml_s = reinterpret_cast<float2*>(red_l + 2 * ATC_BQ);  // [128] (max, sum) of this chunk
  float* osm = reinterpret_cast<float*>(sK);                     // [128][OS_LD] scaled O, after all MMAs

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.Hq / p.Hkv;
  const int b = blockIdx.y / p.Hkv, kvh = blockIdx.y % p.Hkv;
  const int rows_total = p.n * G;
  const int row_base = blockIdx.x * ATC_BQ;
  int kend_cta;
  if (p.causal) {
    const int i_last = min((row_base + ATC_BQ - 1) / G, p.n - 1);
    kend_cta = p.pos0 + i_last + 1;
  } else {
    kend_cta = p.pos0 + p.n;
  }
  const int kbeg = blockIdx.z * p.chunk_len;
  const int kend = min(kbeg + p.chunk_len, kend_cta);
  const int nb = kend > kbeg ? (kend - kbeg + ATC_BK - 1) / ATC_BK : 0;
  const int kv_row0 = (b * p.Hkv + kvh) * p.S_max + kbeg;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < ATC_KSTAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < ATC_VSTAGES; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 128);
      mbar_init(&p_full[s], 128);
      mbar_init(&p_empty[s], 1);
    }
    mbar_init(o_full, 1);
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
  const int wg = (warp - 2) >> 2;                // softmax warpgroup 0 / 1
  const int quarter = warp & 3;                  // TMEM lanes this warp may access
  const int rloc = quarter * 32 + lane;          // packed row of the tile = TMEM lane
  const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
  const int r = row_base + rloc;
  const bool live = r < rows_total;
  float mref = -INFINITY, lsum = 0.f;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0 && nb > 0) {
      tma_prefetch_desc(&p.q_map);
      tma_prefetch_desc(&p.k_map);
      tma_prefetch_desc(&p.v_map);
      const uint64_t pol = policy_evict_last();  // K/V blocks are shared by the head's query blocks
      uint32_t k_issued = 0, k_par = 0, v_issued = 0, v_par = 0;
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
      for (int db = 0; db < C::DK; ++db)
        tma_load_4d(sQ + db * ATC_BQ * 128, &p.q_map, q_full, db * 64, 0, kvh, b * p.n + row_base / G, pol);
      int uk = 0, uv = 0;
      for (int pass = 0; pass < 2 && !*abort_flag; ++pass) {
        for (int j = 0; j < nb; ++j) {
          const int s = uk % ATC_KSTAGES;
          const uint32_t ph = (uk / ATC_KSTAGES) & 1;
          if (!mbar_wait(&k_empty[s], ph ^ 1, p.err)) {
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(&k_full[s], C::KV_BYTES);
          for (int db = 0; db < C::DK; ++db)
            tma_load_2d(sK + s * C::KV_BYTES + db * ATC_BK * 128, &p.k_map, &k_full[s], db * 64,
                        kv_row0 + j * ATC_BK, pol);
          k_issued |= 1u << s;
          k_par = (k_par & ~(1u << s)) | (ph << s);
          ++uk;
          if (pass == 1) {
            const int sv = uv % ATC_VSTAGES;
            const uint32_t phv = (uv / ATC_VSTAGES) & 1;
            if (!mbar_wait(&v_empty[sv], phv ^ 1, p.err)) {
              *abort_flag = 1;
              break;
            }
            mbar_arrive_expect_tx(&v_full[sv], C::KV_BYTES);
            for (int db = 0; db < C::DK; ++db)
              tma_load_2d(sV + sv * C::KV_BYTES + db * ATC_BK * 128, &p.v_map, &v_full[sv], db * 64,
                          kv_row0 + j * ATC_BK, pol);
            v_issued |= 1u << sv;
            v_par = (v_par & ~(1u << sv)) | (phv << sv);
            ++uv;
          }
        }
      }
      // every copy issued here has landed before its buffer is reused or the CTA exits
      mbar_wait(q_full, 0, p.err);
      for (int s = 0; s < ATC_KSTAGES; ++s)
        if ((k_issued >> s) & 1) mbar_wait(&k_full[s], (k_par >> s) & 1, p.err);
      for (int s = 0; s < ATC_VSTAGES; ++s)
        if ((v_issued >> s) & 1) mbar_wait(&v_full[s], (v_par >> s) & 1, p.err);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0 && nb > 0) {
      constexpr uint32_t IDESC_S = umma_idesc_bf16(ATC_BQ, ATC_BK);             // Q, K both K-major
      constexpr uint32_t IDESC_PV = umma_idesc_bf16(ATC_BQ, D) | (1u << 16);    // V is MN-major
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV), p_addr = smem_u32(sP);
      // S tile u (u < nb: pass 1, block u; u >= nb: pass 2, block u - nb) into TMEM buffer u & 1
      auto issue_s = [&](int u) -> bool {
        const int sb = u & 1, ks = u % ATC_KSTAGES;
        if (!mbar_wait(&s_empty[sb], ((u >> 1) & 1) ^ 1, p.err)) return false;
        if (!mbar_wait(&k_full[ks], (u / ATC_KSTAGES) & 1, p.err)) return false;
        tc_fence_after();
        const uint32_t kb = k_addr + ks * C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t a_at = q_addr + (kk >> 2) * (ATC_BQ * 128) + (kk & 3) * 32;
          const uint32_t b_at = kb + (kk >> 2) * (ATC_BK * 128) + (kk & 3) * 32;
          umma_bf16(tmem_base + sb * ATC_BK, umma_desc_sw128(a_at), umma_desc_sw128(b_at), IDESC_S,
                    kk > 0 ? 1u : 0u);
        }
        umma_commit(&k_empty[ks]);
        umma_commit(&s_full[sb]);
        return true;
      };
      // O += P_j V_j (P buffer j & 1, written by the warpgroup that owns S tile nb + j)
      auto issue_pv = [&](int j) -> bool {
        const int vs = j % ATC_VSTAGES, pb = j & 1;
        if (!mbar_wait(&v_full[vs], (j / ATC_VSTAGES) & 1, p.err)) return false;
        if (!mbar_wait(&p_full[pb], (j >> 1) & 1, p.err)) return false;
        tc_fence_after();
        const uint32_t vb = v_addr + vs * C::KV_BYTES, pbuf = p_addr + pb * C::P_BYTES;
#pragma unroll
        for (int kk = 0; kk < ATC_BK / 16; ++kk)
          umma_bf16(tmem_base + C::O_COL, umma_desc_sw128(pbuf + kk * 32),
                    umma_desc_sw128_mn(vb + kk * 2048, ATC_BK * 128), IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&v_empty[vs]);
        umma_commit(&p_empty[pb]);
        return true;
      };
      bool mok = mbar_wait(q_full, 0, p.err);
      tc_fence_after();
      for (int u = 0; u < nb && mok; ++u) mok = issue_s(u);
      // pass 2 keeps two S tiles ahead of the P V products: the tile for block
      // j + 2 reuses the buffer that block j's warpgroup released before it
      // produced P_j, so issuing it right after P_j V_j never waits
      if (mok) mok = issue_s(nb);
      if (mok && nb > 1) mok = issue_s(nb + 1);
      for (int j = 0; j < nb && mok; ++j) {
        mok = issue_pv(j);
        if (mok && j + 2 < nb) mok = issue_s(nb + j + 2);
        if (*abort_flag) mok = false;
      }
      if (mok) umma_commit(o_full);
      if (!mok) *abort_flag = 1;
      // every MMA issued has completed before TMEM or its operands are reused
      umma_commit(drain);
      mbar_wait(drain, 0, p.err);
    }
  } else {
    // ----------------------- softmax warpgroups (warps 2..9) -----------------------
    const int i = live ? r / G : 0;
    // keys of this chunk the row sees: [0, lim) relative to kbeg
    const int lim = (live ? min(p.causal ? p.pos0 + i + 1 : p.pos0 + p.n, kend) : 0) - kbeg;
    float s[64];
    // pass 1: row maximum of the raw scores over this warpgroup's S tiles
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    for (int u = wg; u < nb && ok; u += 2) {
      // warp-uniform decision: tcgen05.ld below is a warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[wg], (u >> 1) & 1, p.err) && !*abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_ld64(t_row + wg * ATC_BK, s);
      tc_fence_before();
      mbar_arrive(&s_empty[wg]);
      const int lj = lim - u * ATC_BK;
      if (lj >= ATC_BK) {
#pragma unroll
        for (int c = 0; c < ATC_BK; ++c) mx[c & 3] = fmaxf(mx[c & 3], s[c]);
      } else {
#pragma unroll
        for (int c = 0; c < ATC_BK; ++c)
          if (c < lj) mx[c & 3] = fmaxf(mx[c & 3], s[c]);
      }
    }
    red_m[wg * ATC_BQ + rloc] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
    named_bar_sync(1, 256);
    // scale > 0, so the maximum of the scaled scores is the scaled maximum
    mref = fmaxf(red_m[rloc], red_m[ATC_BQ + rloc]) * p.scale_log2;
    // pass 2: P = 2^(s * scale - max) in bf16 to shared memory, row sums
    float l = 0.f;
    for (int j = (wg + nb) & 1; j < nb && ok; j += 2) {
      const int u = nb + j, pb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[wg], (u >> 1) & 1, p.err) && !*abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_ld64(t_row + wg * ATC_BK, s);
      tc_fence_before();
      mbar_arrive(&s_empty[wg]);
      const int lj = lim - j * ATC_BK;
      uint32_t pk[ATC_BK / 2];
#pragma unroll
      for (int c = 0; c < ATC_BK / 2; ++c) {
        const float p0 = (2 * c < lj) ? ex2_approx(fmaf(s[2 * c], p.scale_log2, -mref)) : 0.f;
        const float p1 = (2 * c + 1 < lj) ? ex2_approx(fmaf(s[2 * c + 1], p.scale_log2, -mref)) : 0.f;
        l += p0 + p1;
        pk[c] = pack_bf16x2(p0, p1);
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&p_empty[pb], ((j >> 1) & 1) ^ 1, p.err))) {
        ok = false;
        break;
      }
      // row rloc of a K-major 128-byte-swizzled tile: 16-byte chunk c lands at c ^ (row & 7)
      uint8_t* dst = sP + pb * C::P_BYTES + rloc * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        *reinterpret_cast<uint4*>(dst + ((ch ^ (rloc & 7)) << 4)) =
            make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      fence_proxy_async_smem();
      mbar_arrive(&p_full[pb]);
    }
    red_l[wg * ATC_BQ + rloc] = l;
    if (!ok) *abort_flag = 1;
    named_bar_sync(1, 256);
    lsum = red_l[rloc] + red_l[ATC_BQ + rloc];
    if (nb > 0 && ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(o_full, 0, p.err) && !*abort_flag);
      tc_fence_after();
    }
    if (nb == 0) mref = -INFINITY;
    if (wg == 0) ml_s[rloc] = make_float2(mref, lsum);
  }

  // ---------- merge the key chunks of this query block (one cluster) ----------
  // o = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c, M = max_c m_c: each chunk
  // scales its own rows into shared memory, then every chunk sums a slice of
  // the rows over all chunks' tiles (distributed shared memory) and stores it.
  const int nc = p.n_chunks;
  cluster_sync_all();  // every chunk's (max, sum) is visible
  if (warp >= 2) {
    const uint32_t ml_at = smem_u32(&ml_s[rloc]);
    float M = -INFINITY;
    for (int q = 0; q < nc; ++q) M = fmaxf(M, ld_dsmem_f2(mapa_shared(ml_at, q)).x);
    const float Mref = M == -INFINITY ? 0.f : M;
    float den = 0.f;
    for (int q = 0; q < nc; ++q) {
      const float2 v = ld_dsmem_f2(mapa_shared(ml_at, q));
      den += v.y * ex2_approx(v.x - Mref);
    }
    const float w = (den > 0.f && mref != -INFINITY) ? ex2_approx(mref - Mref) / den : 0.f;
    const bool have_o = nb > 0 && ok;  // warp-uniform
#pragma unroll
    for (int k = wg; k < D / 16; k += 2) {
      float v[16];
      if (have_o) {
        tmem_ld16(t_row + C::O_COL + k * 16, v);
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = 0.f;
      }
      float4* dst = reinterpret_cast<float4*>(osm + rloc * C::OS_LD + k * 16);
#pragma unroll
      for (int e = 0; e < 4; ++e) dst[e] = make_float4(v[4 * e] * w, v[4 * e + 1] * w, v[4 * e + 2] * w, v[4 * e + 3] * w);
    }
  }
  cluster_sync_all();  // every chunk's scaled tile is complete
  if (warp >= 2) {
    const int rank = static_cast<int>(cluster_ctarank());
    const int rpr = (ATC_BQ + nc - 1) / nc;
    const int r_lo = rank * rpr, r_hi = min(ATC_BQ, r_lo + rpr);
    constexpr int D4 = D / 4;
    const uint32_t os_at = smem_u32(osm);
    // two items per pass, all their peer loads issued before any is used
    const int n_items = (r_hi - r_lo) * D4;
    for (int it0 = threadIdx.x - 64; it0 < n_items; it0 += 512) {
      float4 acc[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
      float4 v[2][ATC_MAX_CHUNKS];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int it = it0 + 256 * h;
        const int rr = r_lo + it / D4, c4 = (it % D4) * 4;
        const uint32_t off = static_cast<uint32_t>((rr * C::OS_LD + c4) * 4);
#pragma unroll
        for (int q = 0; q < ATC_MAX_CHUNKS; ++q)
          if (q < nc && it < n_items) v[h][q] = ld_dsmem_f4(mapa_shared(os_at + off, q));
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int it = it0 + 256 * h;
        if (it >= n_items) continue;
#pragma unroll
        for (int q = 0; q < ATC_MAX_CHUNKS; ++q)
          if (q < nc) {
            acc[h].x += v[h][q].x;
            acc[h].y += v[h][q].y;
            acc[h].z += v[h][q].z;
            acc[h].w += v[h][q].w;
          }
        const int rr = r_lo + it / D4, c4 = (it % D4) * 4;
        const int rg = row_base + rr;
        if (rg >= rows_total) continue;
        const size_t rid = (static_cast<size_t>(b) * p.n + rg / G) * p.Hq + kvh * G + rg % G;
        *reinterpret_cast<uint2*>(p.o + rid * D + c4) =
            make_uint2(pack_bf16x2(acc[h].x, acc[h].y), pack_bf16x2(acc[h].z, acc[h].w));
      }
    }
  }
  cluster_sync_all();  // no CTA leaves while a peer may still read its shared memory

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace dg
