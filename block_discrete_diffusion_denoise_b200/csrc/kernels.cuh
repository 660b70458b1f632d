// Memory-bound kernels of the step: embedding gather + RMSNorm, split-K
// reduction + residual + RMSNorm, QKV reduction + RoPE + KV write, router
// top-k, token permutation and expert tile lists, row gather, gate-weighted
// combine + residual + RMSNorm, LM-head partial merge + Philox sampler.
#pragma once

#include "common.cuh"

namespace dg {

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., SC'11): 4-word counter, 2-word key, ten rounds
// of two 32x32->64 multiplies with the key bumped by the Weyl constants.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k.x += 0x9E3779B9u;
      k.y += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
  }
  return c;
}

__device__ __forceinline__ int uniform_token(uint32_t w, int vocab) {
  if ((vocab & (vocab - 1)) == 0) return static_cast<int>(w & static_cast<uint32_t>(vocab - 1));
  return static_cast<int>((static_cast<uint64_t>(w) * static_cast<uint64_t>(vocab)) >> 32);
}

// Router: logits = sum_s part[s][row][e] (+ bias[e]); top-k by (logit desc,
// index asc); gates = softmax over the k selected.  One warp per row; CTA c
// owns rows [c * rows_per_cta, (c + 1) * rows_per_cta).  With `counts`, the
// (row, slot) pairs choosing each expert are added to counts[e] (zero before
// the launch).
constexpr int PERM_MAXE = 256;

__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ part, int splits, int T, int E,
                                                          int k, const float* __restrict__ bias,
                                                          int32_t* __restrict__ idx_out,
                                                          float* __restrict__ gates_out,
                                                          int32_t* __restrict__ capture, int rows_per_cta,
                                                          int32_t* __restrict__ counts) {
  __shared__ int s_hist[PERM_MAXE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (counts) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
    __syncthreads();
  }
  const int row_end = min(T, (blockIdx.x + 1) * rows_per_cta);
  for (int row = blockIdx.x * rows_per_cta + warp; row < row_end; row += blockDim.x >> 5) {
    constexpr int MAXPER = PERM_MAXE / 32;
    float v[MAXPER];
    uint32_t taken = 0;
#pragma unroll
    for (int c = 0; c < MAXPER; ++c) {
      const int e = c * 32 + lane;
      float x = -INFINITY;
      if (e < E) {
        x = 0.f;
        for (int s = 0; s < splits; ++s) x += part[(static_cast<size_t>(s) * T + row) * E + e];
        if (bias) x += bias[e];
      }
      v[c] = x;
    }
    // lane r keeps the r-th selection (k <= 16 < 32)
    float my_v = -INFINITY, top_v = -INFINITY;
    int my_i = 0;
    for (int r = 0; r < k; ++r) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int c = 0; c < MAXPER; ++c) {
        const int e = c * 32 + lane;
        if (e < E && !((taken >> c) & 1) && (v[c] > bv || (v[c] == bv && e < bi) || bi == 0x7fffffff)) {
          bv = v[c];
          bi = e;
        }
      }
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
          bv = ov;
          bi = oi;
        }
      }
      if (r == 0) top_v = bv;
      if (lane == r) {
        my_v = bv;
        my_i = bi;
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    }
    // gates: softmax over the k selected logits, summed in slot order
    const float w = lane < k ? __expf(my_v - top_v) : 0.f;
    float sum = 0.f;
    for (int r = 0; r < k; ++r) sum += __shfl_sync(0xffffffffu, w, r);
    if (lane < k) {
      idx_out[static_cast<size_t>(row) * k + lane] = my_i;
      gates_out[static_cast<size_t>(row) * k + lane] = w / sum;
      if (capture) capture[static_cast<size_t>(row) * k + lane] = my_i;
      if (counts) atomicAdd(&s_hist[my_i], 1);
    }
  }
  if (counts) {
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
      if (s_hist[e] > 0) atomicAdd(&counts[e], s_hist[e]);
  }
}

// exclusive scan over the 256 threads of a block; `tmp` >= 8 ints
__device__ __forceinline__ int block_excl_scan256(int v, int* tmp, int& total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  int wbase = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const int t = tmp[w];
    if (w < warp) wbase += t;
    total += t;
  }
  __syncthreads();
  return wbase + x - v;
}

// Permutation of the T*k (row, slot) pairs by expert, the gather of the
// routed rows, and the tile list of the fused expert GEMM.  Expert e owns
// positions [start_e, start_e + counts[e]); pairs claim positions in it from
// cursor[e].  The order of rows within an expert does not change any value
// (every row of a tile is an independent dot product and the combine sums a
// token's slots in slot order through inv_slot), so the claim order is free.
//   perm_tok[pos]   row of permuted position pos;  xp[pos] = u[perm_tok[pos]]
//   inv_slot[p]     permuted position of pair p = t*k + j
//   tiles           gate/up tiles, then down tiles, each
//                   {group | block << 16, token chunk, first row, rows};
//                   groups in the order shared (= E, all T rows), 0, ..., E-1;
//                   within a group block-major, so re-reads of a weight block
//                   by its chunks hit L2
//   chunk_done[c]   zeroed (gate/up tiles of chunk c finished)
//   counters[0] = gate/up tiles, [1] = down tiles, [2] = experts hit,
//   counters[3] = tile claim counter (zeroed)
//   route[0..E) = counts, route[E..2E) = cursors, route[2E] = finished CTAs:
//   the last CTA to finish zeroes them for the next launch.
__global__ void __launch_bounds__(256) permute_gather_kernel(
    const int32_t* __restrict__ idx, int32_t* __restrict__ route, int rows_per_cta, int T, int k, int E, int F,
    int Fs, int d, const uint16_t* __restrict__ u, int32_t* __restrict__ perm_tok, int32_t* __restrict__ inv_slot,
    uint16_t* __restrict__ xp, int4* __restrict__ tiles, int32_t* __restrict__ chunk_done,
    int32_t* __restrict__ counters, int chunk_rows) {
  __shared__ int s_start[PERM_MAXE];   // first position of each expert
  __shared__ int s_cnt[PERM_MAXE];
  __shared__ int s_pos[256];
  __shared__ int tmp[8];
  __shared__ int s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t* cursor = route + E;
  {
    const int c = threadIdx.x < E ? __ldcg(&route[threadIdx.x]) : 0;
    int total;
    const int ex = block_excl_scan256(c, tmp, total);
    if (threadIdx.x < E) {
      s_start[threadIdx.x] = ex;
      s_cnt[threadIdx.x] = c;
    }
  }
  __syncthreads();

  if (blockIdx.x == 0) {
    // Tile list.  Slot s = 0 is the shared expert, slot s >= 1 expert s - 1;
    // each thread takes slots 2t and 2t + 1 of the scans.
    const int mb_dn = d / 128;
    int nch[2], gu[2], dn[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int sl = 2 * threadIdx.x + h;
      const int cnt = sl == 0 ? T : (sl <= E ? s_cnt[sl - 1] : 0);
      nch[h] = (cnt + chunk_rows - 1) / chunk_rows;
      gu[h] = nch[h] * ((sl == 0 ? Fs : F) / 64);
      dn[h] = nch[h] * mb_dn;
    }
    int tot_ch, tot_gu, tot_dn;
    const int ch0 = block_excl_scan256(nch[0] + nch[1], tmp, tot_ch);
    const int gu0 = block_excl_scan256(gu[0] + gu[1], tmp, tot_gu);
    const int dn0 = block_excl_scan256(dn[0] + dn[1], tmp, tot_dn);
    const int hit = __syncthreads_count(threadIdx.x < E && s_cnt[threadIdx.x] > 0) +
                    __syncthreads_count(threadIdx.x + 256 < E && s_cnt[threadIdx.x + 256] > 0);
    if (threadIdx.x == 0) {
      counters[0] = tot_gu;
      counters[1] = tot_dn;
      counters[2] = hit;
      counters[3] = 0;
    }
    for (int c = threadIdx.x; c < tot_ch; c += 256) chunk_done[c] = 0;
    int ch_at = ch0, gu_at = gu0, dn_at = tot_gu + dn0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int sl = 2 * threadIdx.x + h;
      if (sl <= E) {
        const int g = sl == 0 ? E : sl - 1;
        const int cnt = sl == 0 ? T : s_cnt[g];
        const int first = sl == 0 ? 0 : s_start[g];
        const int mb_gu = (sl == 0 ? Fs : F) / 64;
        for (int j = 0; j < mb_gu; ++j)
          for (int ch = 0; ch < nch[h]; ++ch)
            tiles[gu_at++] = make_int4(g | (j << 16), ch_at + ch, first + ch * chunk_rows,
                                       min(chunk_rows, cnt - ch * chunk_rows));
        for (int j = 0; j < mb_dn; ++j)
          for (int ch = 0; ch < nch[h]; ++ch)
            tiles[dn_at++] = make_int4(g | (j << 16), ch_at + ch, first + ch * chunk_rows,
                                       min(chunk_rows, cnt - ch * chunk_rows));
        ch_at += nch[h];
      }
    }
  }

  // positions of this CTA's pairs, 256 at a time (one warp-aggregated claim
  // per expert and warp), then the gather of their rows
  const unsigned lt = (1u << lane) - 1u;
  const int p_begin = blockIdx.x * rows_per_cta * k;
  const int p_end = min(T, (blockIdx.x + 1) * rows_per_cta) * k;
  const int vec = d / 8;
  for (int c0 = p_begin; c0 < p_end; c0 += 256) {
    const int p = c0 + threadIdx.x;
    const bool valid = p < p_end;
    const int e = valid ? idx[p] : -1;
    const unsigned m = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(m) - 1;
    int base = 0;
    if (valid && lane == leader) base = atomicAdd(&cursor[e], __popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (valid) {
      const int pos = s_start[e] + base + __popc(m & lt);
      perm_tok[pos] = p / k;
      inv_slot[p] = pos;
      s_pos[threadIdx.x] = pos;
    }
    __syncthreads();
    // one warp per pair; each lane keeps 4 row loads in flight
    const int n_here = min(256, p_end - c0);
    for (int pr = warp; pr < n_here; pr += 8) {
      const uint4* src = reinterpret_cast<const uint4*>(u) + static_cast<size_t>((c0 + pr) / k) * vec;
      uint4* dst = reinterpret_cast<uint4*>(xp) + static_cast<size_t>(s_pos[pr]) * vec;
      for (int cv = lane; cv < vec; cv += 128) {
        uint4 r[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (cv + 32 * q < vec) r[q] = src[cv + 32 * q];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (cv + 32 * q < vec) dst[cv + 32 * q] = r[q];
      }
    }
    __syncthreads();
  }

  // the last CTA out zeroes the counts and cursors (every CTA has read the
  // counts and made its claims before it counts itself out)
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&route[2 * E], 1) == static_cast<int>(gridDim.x) - 1;
  __syncthreads();
  if (s_last) {
    for (int e = threadIdx.x; e < 2 * E; e += 256) route[e] = 0;
    __syncthreads();
    if (threadIdx.x == 0) route[2 * E] = 0;
  }
}

// ---------------------------------------------------------------------------
// Row kernels: one CTA of ROW_THREADS per row; each thread keeps up to
// ROW_MAXV float4 of the row in registers between the update and the norm.
// ---------------------------------------------------------------------------
constexpr int ROW_THREADS = 256;
constexpr int ROW_MAXV = 4;  // d <= ROW_THREADS * ROW_MAXV * 4 = 4096

__device__ __forceinline__ float4 load_bf16x4(const uint16_t* src) {
  const uint2 i = *reinterpret_cast<const uint2*>(src);
  return make_float4(bf16_to_f32(static_cast<uint16_t>(i.x & 0xffffu)), bf16_to_f32(static_cast<uint16_t>(i.x >> 16)),
                     bf16_to_f32(static_cast<uint16_t>(i.y & 0xffffu)), bf16_to_f32(static_cast<uint16_t>(i.y >> 16)));
}

__device__ __forceinline__ void store_bf16x4(uint16_t* dst, float4 v) {
  uint2 o;
  o.x = pack_bf16x2(v.x, v.y);
  o.y = pack_bf16x2(v.z, v.w);
  *reinterpret_cast<uint2*>(dst) = o;
}

__device__ __forceinline__ float4 f4_add(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

__device__ __forceinline__ float4 f4_fma(float s, float4 a, float4 b) {  // b + s * a
  return make_float4(fmaf(s, a.x, b.x), fmaf(s, a.y, b.y), fmaf(s, a.z, b.z), fmaf(s, a.w, b.w));
}

__device__ __forceinline__ float f4_sumsq(float4 a) { return a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w; }

// u_row = RMSNorm(row held in v) * gain, as bf16
__device__ __forceinline__ void norm_store_row(const float4 (&v)[ROW_MAXV], float ss, int d,
                                               const uint16_t* __restrict__ gain, float eps,
                                               uint16_t* __restrict__ urow, float* red) {
  ss = block_sum(ss, red);
  const float r = rsqrtf(ss / d + eps);
  const int nv = d / 4;
#pragma unroll
  for (int i = 0; i < ROW_MAXV; ++i) {
    const int c = threadIdx.x + i * ROW_THREADS;
    if (c < nv) {
      const float4 g = load_bf16x4(gain + 4 * c);
      const float4 x = v[i];
      store_bf16x4(urow + 4 * c, make_float4(x.x * r * g.x, x.y * r * g.y, x.z * r * g.z, x.w * r * g.w));
    }
  }
}

// h[t] += y_shared[t] + sum_j gate[t][j] * y[inv_slot[t][j]] (in that order);
// u = RMSNorm(h) * gain
__global__ void __launch_bounds__(ROW_THREADS) combine_norm_kernel(
    float* __restrict__ h, const float* __restrict__ yp, const int32_t* __restrict__ inv_slot,
    const float* __restrict__ gates, int k, int shared_base, int d, const uint16_t* __restrict__ gain, float eps,
    uint16_t* __restrict__ u, float* __restrict__ capture) {
  __shared__ float red[32];
  __shared__ int slot[16];
  __shared__ float gw[16];
  const int row = blockIdx.x;
  if (threadIdx.x < k) {
    slot[threadIdx.x] = inv_slot[static_cast<size_t>(row) * k + threadIdx.x];
    gw[threadIdx.x] = gates[static_cast<size_t>(row) * k + threadIdx.x];
  }
  __syncthreads();
  const int nv = d / 4;
  float4* hrow = reinterpret_cast<float4*>(h + static_cast<size_t>(row) * d);
  const float4* ys = reinterpret_cast<const float4*>(yp + static_cast<size_t>(shared_base + row) * d);
  float4 v[ROW_MAXV];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < ROW_MAXV; ++i) {
    const int c = threadIdx.x + i * ROW_THREADS;
    if (c < nv) {
      float4 x = f4_add(hrow[c], ys[c]);
      for (int s = 0; s < k; ++s)
        x = f4_fma(gw[s], reinterpret_cast<const float4*>(yp + static_cast<size_t>(slot[s]) * d)[c], x);
      hrow[c] = x;
      if (capture) reinterpret_cast<float4*>(capture + static_cast<size_t>(row) * d)[c] = x;
      v[i] = x;
      ss += f4_sumsq(x);
    }
  }
  norm_store_row(v, ss, d, gain, eps, u + static_cast<size_t>(row) * d, red);
}

// Embedding gather (bf16 -> fp32 residual) + RMSNorm -> bf16.
// Token of row b*n+i: tokens[b * tok_stride + tok_off + i]; ids outside the
// vocabulary are clamped into it rather than read out of bounds.
__global__ void __launch_bounds__(ROW_THREADS) embed_norm_kernel(
    const int32_t* __restrict__ tokens, int tok_stride, int tok_off, int n, const uint16_t* __restrict__ embed,
    const uint16_t* __restrict__ gain, float eps, int d, float* __restrict__ h, uint16_t* __restrict__ u,
    float* __restrict__ capture, int32_t* settled, int n_settled, int vocab) {
  __shared__ float red[32];
  const int row = blockIdx.x;
  const int b = row / n, i = row % n;
  if (settled != nullptr && row == 0 && threadIdx.x < n_settled) settled[threadIdx.x] = 1;
  const int tok = min(max(tokens[static_cast<size_t>(b) * tok_stride + tok_off + i], 0), vocab - 1);
  const uint16_t* e = embed + static_cast<size_t>(tok) * d;
  float4* hrow = reinterpret_cast<float4*>(h + static_cast<size_t>(row) * d);
  const int nv = d / 4;
  float4 v[ROW_MAXV];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < ROW_MAXV; ++j) {
    const int c = threadIdx.x + j * ROW_THREADS;
    if (c < nv) {
      const float4 x = load_bf16x4(e + 4 * c);
      hrow[c] = x;
      if (capture) reinterpret_cast<float4*>(capture + static_cast<size_t>(row) * d)[c] = x;
      v[j] = x;
      ss += f4_sumsq(x);
    }
  }
  norm_store_row(v, ss, d, gain, eps, u + static_cast<size_t>(row) * d, red);
}

// h[row] += sum_s part[s][row] (splits in order); u[row] = RMSNorm(h[row]) * gain
__global__ void __launch_bounds__(ROW_THREADS) residual_norm_kernel(
    float* __restrict__ h, const float* __restrict__ part, int splits, int T, int d,
    const uint16_t* __restrict__ gain, float eps, uint16_t* __restrict__ u) {
  __shared__ float red[32];
  const int row = blockIdx.x;
  const int nv = d / 4;
  float4* hrow = reinterpret_cast<float4*>(h + static_cast<size_t>(row) * d);
  float4 v[ROW_MAXV];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < ROW_MAXV; ++j) {
    const int c = threadIdx.x + j * ROW_THREADS;
    if (c < nv) {
      float4 x = hrow[c];
      for (int s = 0; s < splits; ++s)
        x = f4_add(x, reinterpret_cast<const float4*>(part + (static_cast<size_t>(s) * T + row) * d)[c]);
      hrow[c] = x;
      v[j] = x;
      ss += f4_sumsq(x);
    }
  }
  norm_store_row(v, ss, d, gain, eps, u + static_cast<size_t>(row) * d, red);
}

// Reduce the QKV split-K partials (splits in order), rotate q and k pairs
// (j, j + D/2) at absolute position pos0 + i, write q [row][Hq][D] bf16 and
// k, v into this layer's cache [B][Hkv][S_max][D] at that position.  Four
// consecutive j per thread (D/2 is a multiple of 4).
__global__ void __launch_bounds__(ROW_THREADS) rope_qkv_kernel(
    const float* __restrict__ part, int splits, int T, int n, int pos0, int Hq, int Hkv, int D,
    const float2* __restrict__ rope_tab, uint16_t* __restrict__ q, uint16_t* __restrict__ kc,
    uint16_t* __restrict__ vc, int S_max) {
  const int row = blockIdx.x;
  const int b = row / n, i = row % n;
  const int pos = pos0 + i;
  const int QKV = (Hq + 2 * Hkv) * D;
  const int half = D / 2, hq4 = half / 4, d4 = D / 4;
  const float* base = part + static_cast<size_t>(row) * QKV;
  const size_t sstride = static_cast<size_t>(T) * QKV;
  const int n_rot = (Hq + Hkv) * hq4;
  for (int it = threadIdx.x; it < n_rot + Hkv * d4; it += ROW_THREADS) {
    if (it < n_rot) {
      const int hh = it / hq4, j = (it % hq4) * 4;
      const int c = hh * D + j;
      float4 x1 = make_float4(0.f, 0.f, 0.f, 0.f), x2 = x1;
      for (int s = 0; s < splits; ++s) {
        x1 = f4_add(x1, *reinterpret_cast<const float4*>(base + s * sstride + c));
        x2 = f4_add(x2, *reinterpret_cast<const float4*>(base + s * sstride + c + half));
      }
      const float2* cs = rope_tab + static_cast<size_t>(pos) * half + j;
      const float2 c0 = cs[0], c1 = cs[1], c2 = cs[2], c3 = cs[3];
      const float4 y1 = make_float4(x1.x * c0.x - x2.x * c0.y, x1.y * c1.x - x2.y * c1.y,
                                    x1.z * c2.x - x2.z * c2.y, x1.w * c3.x - x2.w * c3.y);
      const float4 y2 = make_float4(x2.x * c0.x + x1.x * c0.y, x2.y * c1.x + x1.y * c1.y,
                                    x2.z * c2.x + x1.z * c2.y, x2.w * c3.x + x1.w * c3.y);
      uint16_t* dst = hh < Hq ? q + (static_cast<size_t>(row) * Hq + hh) * D
                              : kc + ((static_cast<size_t>(b) * Hkv + (hh - Hq)) * S_max + pos) * D;
      store_bf16x4(dst + j, y1);
      store_bf16x4(dst + j + half, y2);
    } else {
      const int r = it - n_rot;
      const int g = r / d4, j = (r % d4) * 4;
      const int c = (Hq + Hkv) * D + g * D + j;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s = 0; s < splits; ++s) x = f4_add(x, *reinterpret_cast<const float4*>(base + s * sstride + c));
      store_bf16x4(vc + ((static_cast<size_t>(b) * Hkv + g) * S_max + pos) * D + j, x);
    }
  }
}

// ---------------------------------------------------------------------------
// LM-head partial merge + sampler.  Partials are in log2 units:
// {m1, argmax, m2, sum 2^(x - m1)} per (vocabulary tile, token).
// ---------------------------------------------------------------------------
struct Top2 {
  float m1;
  int idx;
  float m2;
  float s;
};

__device__ __forceinline__ Top2 top2_merge(Top2 a, Top2 b) {
  if (b.m1 == -INFINITY) return a;
  if (a.m1 == -INFINITY) return b;
  if (b.m1 > a.m1 || (b.m1 == a.m1 && b.idx < a.idx)) {
    const Top2 t = a;
    a = b;
    b = t;
  }
  Top2 r;
  r.m1 = a.m1;
  r.idx = a.idx;
  r.m2 = fmaxf(a.m2, b.m1);
  r.s = a.s + b.s * exp2f(b.m1 - a.m1);
  return r;
}

struct SampleArgs {
  int n_vtiles, T, C, P, step, vocab;
  uint32_t seed_lo, seed_hi;
  float tau;
  int32_t* canvas_out;
  float* conf_out;
  int32_t* settled;
  int32_t* dbg_argmax;
  float* dbg_lse;
  float* dbg_conf;
  float* dbg_margin;
};

__device__ __forceinline__ int sample_decision(int argmax, float conf, float tau, int pos, int step, int seq,
                                               uint32_t seed_lo, uint32_t seed_hi, int vocab) {
  if (conf >= tau) return argmax;  // NaN re-noises
  const uint4 r = philox4x32_10(make_uint4(static_cast<uint32_t>(pos), static_cast<uint32_t>(step),
                                           static_cast<uint32_t>(seq), 0u),
                                make_uint2(seed_lo, seed_hi));
  return uniform_token(r.x, vocab);
}

__global__ void lmhead_merge_sample_kernel(const float4* __restrict__ part, SampleArgs a) {
  __shared__ Top2 sh[32];
  const int t = blockIdx.x;
  Top2 acc{-INFINITY, 0x7fffffff, -INFINITY, 0.f};
  for (int v = threadIdx.x; v < a.n_vtiles; v += blockDim.x) {
    const float4 p = part[static_cast<size_t>(v) * a.T + t];
    acc = top2_merge(acc, Top2{p.x, __float_as_int(p.y), p.z, p.w});
  }
  for (int o = 16; o > 0; o >>= 1) {
    Top2 other;
    other.m1 = __shfl_xor_sync(0xffffffffu, acc.m1, o);
    other.idx = __shfl_xor_sync(0xffffffffu, acc.idx, o);
    other.m2 = __shfl_xor_sync(0xffffffffu, acc.m2, o);
    other.s = __shfl_xor_sync(0xffffffffu, acc.s, o);
    acc = top2_merge(acc, other);
  }
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (blockDim.x >> 5); ++w) acc = top2_merge(acc, sh[w]);
    const float conf = 1.f / acc.s;                      // exp(m1 - lse)
    const float lse = (acc.m1 + log2f(acc.s)) * 0.69314718055994531f;
    const float margin = (1.f - exp2f(acc.m2 - acc.m1)) / acc.s;
    const int b = t / a.C, i = t % a.C;
    const int out = sample_decision(acc.idx, conf, a.tau, a.P + i, a.step, b, a.seed_lo, a.seed_hi, a.vocab);
    a.canvas_out[t] = out;
    if (a.conf_out) a.conf_out[t] = conf;
    if (a.settled && !(conf >= a.tau)) a.settled[b] = 0;
    if (a.dbg_argmax) a.dbg_argmax[t] = acc.idx;
    if (a.dbg_lse) a.dbg_lse[t] = lse;
    if (a.dbg_conf) a.dbg_conf[t] = conf;
    if (a.dbg_margin) a.dbg_margin[t] = margin;
  }
}

// sampler alone (test hook): given argmax / conf
__global__ void sample_only_kernel(const int32_t* __restrict__ argmax, const float* __restrict__ conf, int T,
                                   int C, int P, int step, uint32_t seed_lo, uint32_t seed_hi, float tau,
                                   int vocab, int32_t* __restrict__ out) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  out[t] = sample_decision(argmax[t], conf[t], tau, P + t % C, step, t / C, seed_lo, seed_hi, vocab);
}

// waits on a barrier that is never signalled; the bounded wait must give up
__global__ void wait_timeout_kernel(DevErr err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, err);
}

}  // namespace dg
