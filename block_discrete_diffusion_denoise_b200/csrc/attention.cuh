// Grouped-query attention of new rows over the KV cache, two masks:
//   causal:        row i (position pos0 + i) sees keys [0, pos0 + i]
//   bidirectional: every row sees keys [0, pos0 + n)   (cache + whole canvas)
// Flash-style online softmax with bf16 mma.sync tensor-core tiles; the query
// heads of one GQA group are packed as rows of one tile so each K/V block is
// loaded once per group.  Keys may be split into chunks across CTAs; chunk
// partials (unnormalised O, running max, running sum) are merged afterwards.
#pragma once

#include "common.cuh"

namespace dg {

struct AttnParams {
  const uint16_t* q;   // [T][Hq][D]
  const uint16_t* kc;  // [B][Hkv][S_max][D] (this layer)
  const uint16_t* vc;
  uint16_t* o;         // [T][Hq][D] (single chunk)
  float* opart;        // [chunks][T*Hq][D]   (several chunks)
  float2* ml;          // [chunks][T*Hq]      (max, sum) in log2 units
  int n;               // new rows per sequence
  int B, Hq, Hkv, S_max;
  int pos0;            // cached rows before the new rows
  int causal;
  int chunk_len;       // keys per chunk (multiple of 64)
  int n_chunks;        // <= ATT_MAX_CHUNKS
  float scale_log2;    // log2(e) / sqrt(D)
  int* qb_count;       // per query block: chunks finished (zero between launches)
};

constexpr int ATT_MAX_CHUNKS = 16;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int sz = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

constexpr int ATT_QROWS = 64;   // packed rows per CTA (4 warps x 16)
constexpr int ATT_KB = 64;      // keys per block

template <int D>
constexpr int att_smem_bytes() {
  return 2 /*stages*/ * 2 /*K,V*/ * ATT_KB * (D + 8) * 2;
}

template <int D>
__global__ void __launch_bounds__(128, 2) attn_kernel(const AttnParams p) {
  constexpr int LDS = D + 8;          // smem row stride (elements): conflict-free ldmatrix
  constexpr int NT = D / 8;           // n8 tiles over the head dimension
  constexpr int KT = D / 16;          // k16 steps over the head dimension
  constexpr int CH = D / 8;           // 16-byte chunks per row
  extern __shared__ __align__(16) uint16_t att_smem[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int G = p.Hq / p.Hkv;
  const int b = blockIdx.y / p.Hkv, kvh = blockIdx.y % p.Hkv;
  const int rows_total = p.n * G;
  const int row_base = blockIdx.x * ATT_QROWS;

  // keys this CTA may need
  int kend_cta;
  if (p.causal) {
    const int i_last = min((row_base + ATT_QROWS - 1) / G, p.n - 1);
    kend_cta = p.pos0 + i_last + 1;
  } else {
    kend_cta = p.pos0 + p.n;
  }
  const int kbeg = blockIdx.z * p.chunk_len;
  const int kend = min(kbeg + p.chunk_len, kend_cta);
  const int nblk = kend > kbeg ? (kend - kbeg + ATT_KB - 1) / ATT_KB : 0;

  // this thread's two rows (g, g + 8 of the warp's 16)
  int lim[2], tok[2], head[2];
  bool live[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = row_base + warp * 16 + g + 8 * h;
    live[h] = r < rows_total;
    const int i = live[h] ? r / G : 0;
    tok[h] = b * p.n + i;
    head[h] = kvh * G + (live[h] ? r % G : 0);
    lim[h] = live[h] ? (p.causal ? p.pos0 + i + 1 : p.pos0 + p.n) : 0;
    lim[h] = min(lim[h], kend);
  }

  // Q fragments straight from global memory
  uint32_t qf[KT][4];
#pragma unroll
  for (int kt = 0; kt < KT; ++kt) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint16_t* qrow = p.q + (static_cast<size_t>(tok[h]) * p.Hq + head[h]) * D;
      const uint32_t x0 = live[h] ? *reinterpret_cast<const uint32_t*>(qrow + kt * 16 + 2 * t4) : 0u;
      const uint32_t x1 = live[h] ? *reinterpret_cast<const uint32_t*>(qrow + kt * 16 + 8 + 2 * t4) : 0u;
      qf[kt][h] = x0;       // a0 (row g) / a1 (row g+8)
      qf[kt][2 + h] = x1;   // a2 / a3
    }
  }

  float o[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};

  const uint16_t* kbase = p.kc + (static_cast<size_t>(b) * p.Hkv + kvh) * p.S_max * D;
  const uint16_t* vbase = p.vc + (static_cast<size_t>(b) * p.Hkv + kvh) * p.S_max * D;
  const uint32_t sm0 = smem_u32(att_smem);
  auto stage_k = [&](int s) { return sm0 + static_cast<uint32_t>((s * 2 + 0) * ATT_KB * LDS * 2); };
  auto stage_v = [&](int s) { return sm0 + static_cast<uint32_t>((s * 2 + 1) * ATT_KB * LDS * 2); };

  auto load_block = [&](int blk, int s) {
    const int k0 = kbeg + blk * ATT_KB;
    for (int c = threadIdx.x; c < ATT_KB * CH; c += 128) {
      const int r = c / CH, cc = c % CH;
      const int key = k0 + r;
      const bool ok = key < kend;
      const size_t off = static_cast<size_t>(ok ? key : 0) * D + cc * 8;
      cp_async16(stage_k(s) + (r * LDS + cc * 8) * 2, kbase + off, ok);
      cp_async16(stage_v(s) + (r * LDS + cc * 8) * 2, vbase + off, ok);
    }
    cp_async_commit();
  };

  if (nblk > 0) load_block(0, 0);
  for (int blk = 0; blk < nblk; ++blk) {
    const int s = blk & 1;
    if (blk + 1 < nblk) {
      load_block(blk + 1, s ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int k0 = kbeg + blk * ATT_KB;

    // S = Q K^T for 16 rows x 64 keys
    float sc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt) {
#pragma unroll
      for (int jp = 0; jp < 4; ++jp) {
        const int krow = jp * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int kcol = kt * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(stage_k(s) + (krow * LDS + kcol) * 2, b0, b1, b2, b3);
        mma_bf16_16816(sc[2 * jp], qf[kt], b0, b1);
        mma_bf16_16816(sc[2 * jp + 1], qf[kt], b2, b3);
      }
    }
    // mask + online softmax (log2 units)
    float corr[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = k0 + j * 8 + 2 * t4 + e;
          float x = sc[j][2 * h + e] * p.scale_log2;
          if (key >= lim[h]) x = -INFINITY;
          sc[j][2 * h + e] = x;
          mx = fmaxf(mx, x);
        }
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mnew = fmaxf(mrow[h], mx);
      const float mref = mnew == -INFINITY ? 0.f : mnew;
      corr[h] = exp2f(mrow[h] - mref);
      mrow[h] = mnew;
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float pv = exp2f(sc[j][2 * h + e] - mref);
          sc[j][2 * h + e] = pv;
          sum += pv;
        }
      }
      lrow[h] = lrow[h] * corr[h] + sum;
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      o[j][0] *= corr[0];
      o[j][1] *= corr[0];
      o[j][2] *= corr[1];
      o[j][3] *= corr[1];
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      a[0] = pack_bf16x2(sc[2 * kk][0], sc[2 * kk][1]);
      a[1] = pack_bf16x2(sc[2 * kk][2], sc[2 * kk][3]);
      a[2] = pack_bf16x2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
      a[3] = pack_bf16x2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        const int vrow = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int vcol = np * 16 + (lane >> 4) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(stage_v(s) + (vrow * LDS + vcol) * 2, b0, b1, b2, b3);
        mma_bf16_16816(o[2 * np], a, b0, b1);
        mma_bf16_16816(o[2 * np + 1], a, b2, b3);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int h = 0; h < 2; ++h) {
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 1);
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 2);
  }
  if (p.n_chunks == 1) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (!live[h]) continue;
      const float inv = lrow[h] > 0.f ? 1.f / lrow[h] : 0.f;
      uint16_t* orow = p.o + (static_cast<size_t>(tok[h]) * p.Hq + head[h]) * D;
#pragma unroll
      for (int j = 0; j < NT; ++j)
        *reinterpret_cast<uint32_t*>(orow + j * 8 + 2 * t4) = pack_bf16x2(o[j][2 * h] * inv, o[j][2 * h + 1] * inv);
    }
  } else {
    const size_t nrows = static_cast<size_t>(p.B) * p.n * p.Hq;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (!live[h]) continue;
      const size_t rid = static_cast<size_t>(tok[h]) * p.Hq + head[h];
      float* orow = p.opart + (blockIdx.z * nrows + rid) * D;
#pragma unroll
      for (int j = 0; j < NT; ++j)
        *reinterpret_cast<float2*>(orow + j * 8 + 2 * t4) = make_float2(o[j][2 * h], o[j][2 * h + 1]);
      if (t4 == 0) p.ml[blockIdx.z * nrows + rid] = make_float2(mrow[h], lrow[h]);
    }
    // The last chunk of this query block to finish merges all of them:
    // o = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c  (chunks in order).
    __shared__ int is_last;
    __shared__ float wgt[ATT_QROWS][ATT_MAX_CHUNKS];
    __threadfence();
    __syncthreads();
    const int qb = blockIdx.y * gridDim.x + blockIdx.x;
    if (threadIdx.x == 0) is_last = atomicAdd(p.qb_count + qb, 1) == p.n_chunks - 1;
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    if (threadIdx.x < ATT_QROWS) {
      const int r = row_base + threadIdx.x;
      if (r < rows_total) {
        const size_t rid = (static_cast<size_t>(b) * p.n + r / G) * p.Hq + kvh * G + r % G;
        float M = -INFINITY;
        for (int c = 0; c < p.n_chunks; ++c) M = fmaxf(M, __ldcg(&p.ml[c * nrows + rid].x));
        const float Mref = M == -INFINITY ? 0.f : M;
        float den = 0.f;
        for (int c = 0; c < p.n_chunks; ++c) {
          const float2 v = __ldcg(&p.ml[c * nrows + rid]);
          const float wv = exp2f(v.x - Mref);
          wgt[threadIdx.x][c] = wv;
          den += v.y * wv;
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        for (int c = 0; c < p.n_chunks; ++c) wgt[threadIdx.x][c] *= inv;
      }
    }
    __syncthreads();
    constexpr int D4 = D / 4;
    for (int it = threadIdx.x; it < ATT_QROWS * D4; it += blockDim.x) {
      const int rr = it / D4, j = (it % D4) * 4;
      const int r = row_base + rr;
      if (r >= rows_total) continue;
      const size_t rid = (static_cast<size_t>(b) * p.n + r / G) * p.Hq + kvh * G + r % G;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int c = 0; c < p.n_chunks; ++c) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(p.opart + (c * nrows + rid) * D + j));
        const float wv = wgt[rr][c];
        acc.x += wv * v.x;
        acc.y += wv * v.y;
        acc.z += wv * v.z;
        acc.w += wv * v.w;
      }
      uint16_t* dst = p.o + rid * D + j;
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    }
    if (threadIdx.x == 0) p.qb_count[qb] = 0;  // ready for the next launch
  }
}

// merge chunk partials: o = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c
__global__ void attn_merge_kernel(const float* __restrict__ opart, const float2* __restrict__ ml, int n_chunks,
                                  int nrows, int D, uint16_t* __restrict__ o) {
  const int rid = blockIdx.x;
  float M = -INFINITY;
  for (int c = 0; c < n_chunks; ++c) M = fmaxf(M, ml[static_cast<size_t>(c) * nrows + rid].x);
  const float Mref = M == -INFINITY ? 0.f : M;
  float den = 0.f;
  for (int c = 0; c < n_chunks; ++c) {
    const float2 v = ml[static_cast<size_t>(c) * nrows + rid];
    den += v.y * exp2f(v.x - Mref);
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  for (int j = threadIdx.x; j < D; j += blockDim.x) {
    float acc = 0.f;
    for (int c = 0; c < n_chunks; ++c) {
      const float2 v = ml[static_cast<size_t>(c) * nrows + rid];
      acc += opart[(static_cast<size_t>(c) * nrows + rid) * D + j] * exp2f(v.x - Mref);
    }
    o[static_cast<size_t>(rid) * D + j] = f32_to_bf16(acc * inv);
  }
}

}  // namespace dg
