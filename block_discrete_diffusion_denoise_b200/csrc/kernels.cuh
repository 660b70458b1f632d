// Memory-bound kernels of the step: embedding gather + RMSNorm, split-K
// reduction + residual + RMSNorm, QKV reduction + RoPE + KV write, router
// top-k with the dispatch of every token's activations to its experts' rows,
// gate-weighted combine + residual + RMSNorm, LM-head partial merge + Philox
// sampler, the entropy-constrained sampler, and the split reductions of the
// self-conditioning layer.
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

constexpr int PERM_MAXE = 256;
constexpr int ROUTE_PER = PERM_MAXE / 32;

// Top-k of one row by ranking, over the CTA: lg[0, E) holds the row's logits
// in shared memory (16-byte aligned, E a multiple of 4).  Each thread takes
// experts e = threadIdx.x, threadIdx.x + blockDim.x, ... and counts the
// experts before e in (logit desc, index asc) order; an expert of rank r < k
// is written to sel_v[r], sel_i[r].  The ranks of distinct (logit, index)
// pairs are distinct, so sel holds exactly the k first in that order.
// Callers synchronise the CTA before (lg written) and after (sel read).
__device__ __forceinline__ void cta_rank_topk(const float* lg, int E, int k, float* sel_v, int* sel_i) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const float v = lg[e];
    int rank = 0;
    for (int j = 0; j < E; j += 4) {
      const float4 w = *reinterpret_cast<const float4*>(lg + j);
      rank += (w.x > v || (w.x == v && j < e)) + (w.y > v || (w.y == v && j + 1 < e)) +
              (w.z > v || (w.z == v && j + 2 < e)) + (w.w > v || (w.w == v && j + 3 < e));
    }
    if (rank < k) {
      sel_v[rank] = v;
      sel_i[rank] = e;
    }
  }
}

// logits of one row from split-K partials part[s][row][e] summed in split
// order, plus the per-expert bias: v[c] is the logit of expert c * 32 + lane
// (-inf past E), PER >= E / 32 per lane
template <int PER>
__device__ __forceinline__ void router_logits_row(const float* __restrict__ part, int splits, int T, int row, int E,
                                                  const float* __restrict__ bias, int lane, float (&v)[PER]) {
  constexpr int MAXS = 8;  // split-K partials (the dense GEMM uses at most 8)
#pragma unroll
  for (int c = 0; c < PER; ++c) v[c] = (c * 32 + lane < E) ? 0.f : -INFINITY;
#pragma unroll
  for (int s = 0; s < MAXS; ++s)
    if (s < splits) {
      float t[PER];
#pragma unroll
      for (int c = 0; c < PER; ++c)
        if (c * 32 + lane < E) t[c] = part[(static_cast<size_t>(s) * T + row) * E + c * 32 + lane];
#pragma unroll
      for (int c = 0; c < PER; ++c)
        if (c * 32 + lane < E) v[c] += t[c];
    }
  if (bias) {
#pragma unroll
    for (int c = 0; c < PER; ++c)
      if (c * 32 + lane < E) v[c] += bias[c * 32 + lane];
  }
}

// gates: softmax over the k selected logits (lane r holds selection r), summed
// in slot order; returns this lane's gate (0 for lanes >= k)
__device__ __forceinline__ float selected_gate(float my_v, float top_v, int k, int lane) {
  const float w = lane < k ? __expf(my_v - top_v) : 0.f;
  float sum = 0.f;
  for (int r = 0; r < k; ++r) sum += __shfl_sync(0xffffffffu, w, r);
  return w / sum;
}

// The routing decision of one row (one CTA, blockDim >= 32): warp 0 sums the
// split-K partials into shared memory, the CTA ranks them, and lane r < k of
// warp 0 receives the r-th selection (my_v, my_i) and its gate (softmax over
// the k selected logits, summed in slot order).
template <int PER>
__device__ __forceinline__ void cta_route_row(const float* __restrict__ part, int splits, int T, int row, int E, int k,
                                              const float* __restrict__ bias, float& my_v, int& my_i, float& g) {
  __shared__ __align__(16) float lg[PERM_MAXE];
  __shared__ float sel_v[32];
  __shared__ int sel_i[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    float v[PER];
    router_logits_row<PER>(part, splits, T, row, E, bias, lane, v);
#pragma unroll
    for (int c = 0; c < PER; ++c)
      if (c * 32 + lane < E) lg[c * 32 + lane] = v[c];
  }
  __syncthreads();
  cta_rank_topk(lg, E, k, sel_v, sel_i);
  __syncthreads();
  my_v = -INFINITY;
  my_i = 0;
  g = 0.f;
  if (warp == 0) {
    if (lane < k) {
      my_v = sel_v[lane];
      my_i = sel_i[lane];
    }
    g = selected_gate(my_v, sel_v[0], k, lane);
  }
}

// Router decision alone (test hook): one CTA per row.
__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ part, int splits, int T, int E,
                                                          int k, const float* __restrict__ bias,
                                                          int32_t* __restrict__ idx_out,
                                                          float* __restrict__ gates_out) {
  DG_TIMELINE_SCOPE(TLK_ROUTER_TOPK);
  const int row = blockIdx.x;
  float my_v, g;
  int my_i;
  cta_route_row<ROUTE_PER>(part, splits, T, row, E, k, bias, my_v, my_i, g);
  if (threadIdx.x < k) {
    idx_out[static_cast<size_t>(row) * k + threadIdx.x] = my_i;
    gates_out[static_cast<size_t>(row) * k + threadIdx.x] = g;
  }
}

// Router decision and dispatch of one layer, one CTA of k warps per token row
// (the same decision as router_topk_kernel).  Expert e owns rows [e * region,
// e * region + rows_e) of the routed buffers (gathered activations xp, hidden
// rows, down outputs); each (row, slot) pair claims the next of them from
// cursor[e], so cursor[e] ends as rows_e (zero before the launch; the expert
// GEMM's last CTA zeroes it again).  The order of rows inside a region is
// free: every row of an expert tile is an independent dot product, and the
// combine sums a token's slots in slot order through inv_slot.  The CTA takes
// the decision (cta_route_row) and lane j of warp 0 claims slot j's row; then
// warp j copies the token's normalised row u[row] (which every warp loaded at
// the start, overlapping the decision) to that row.
//   idx, gates [T, k]; inv_slot[row * k + j] = claimed row of slot j;
//   capture [T, k] or NULL (test hook).  blockDim = 32 * k, PER >= E / 32.
constexpr int DISPATCH_MAXV = 16;  // 16-byte chunks per lane: d <= 32 * 16 * 8 = 4096

template <int PER>
__global__ void __launch_bounds__(512) route_dispatch_kernel(
    const float* __restrict__ part, int splits, int T, int E, int k, const float* __restrict__ bias,
    int32_t* __restrict__ idx_out, float* __restrict__ gates_out, int32_t* __restrict__ capture,
    int32_t* __restrict__ cursor, int region, int d, const uint16_t* __restrict__ u, uint16_t* __restrict__ xp,
    int32_t* __restrict__ inv_slot) {
  DG_TIMELINE_SCOPE(TLK_ROUTE_DISPATCH);
  __shared__ int dest[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x;
  const int vec = d / 8;
  const uint4* src = reinterpret_cast<const uint4*>(u) + static_cast<size_t>(row) * vec;
  uint4 x[DISPATCH_MAXV];
#pragma unroll
  for (int i = 0; i < DISPATCH_MAXV; ++i)
    if (lane + 32 * i < vec) x[i] = src[lane + 32 * i];
  float my_v, g;
  int my_i;
  cta_route_row<PER>(part, splits, T, row, E, k, bias, my_v, my_i, g);
  if (threadIdx.x < k) {
    const size_t pr = static_cast<size_t>(row) * k + lane;
    idx_out[pr] = my_i;
    gates_out[pr] = g;
    if (capture) capture[pr] = my_i;
    const int dr = my_i * region + atomicAdd(&cursor[my_i], 1);
    inv_slot[pr] = dr;
    dest[lane] = dr;
  }
  __syncthreads();
  if (warp < k) {
    uint4* dst = reinterpret_cast<uint4*>(xp) + static_cast<size_t>(dest[warp]) * vec;
#pragma unroll
    for (int i = 0; i < DISPATCH_MAXV; ++i)
      if (lane + 32 * i < vec) dst[lane + 32 * i] = x[i];
  }
}

// ---------------------------------------------------------------------------
// Row kernels: one CTA per row, one float4 of the row per thread (blockDim =
// row_threads(d), d <= 4096).  Every load a thread needs is issued before the
// first one is used (split and slot counts are unrolled to their maxima and
// predicated), so a kernel costs a couple of memory round trips.  Sums are
// taken in the same fixed order as before: results are deterministic.
// ---------------------------------------------------------------------------
constexpr int ROW_MAX_SPLITS = 8;  // split-K partials a row kernel sums
constexpr int ROW_MAX_K = 16;      // routed slots the combine sums (in batches of eight)

__host__ __device__ constexpr int row_threads(int d) { return ((d / 4 + 31) / 32) * 32; }

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

// urow = RMSNorm(row) * gain as bf16, x being this thread's float4 (valid: c < d/4)
__device__ __forceinline__ void norm_store_row(float4 x, float4 g, bool valid, int d, float eps,
                                               uint16_t* __restrict__ urow, float* red) {
  const float ss = block_sum(valid ? f4_sumsq(x) : 0.f, red);
  const float r = rsqrtf(ss / d + eps);
  if (valid) store_bf16x4(urow + 4 * threadIdx.x, make_float4(x.x * r * g.x, x.y * r * g.y, x.z * r * g.z, x.w * r * g.w));
}

// h[t] += y_shared[t] + sum_j gate[t][j] * y[inv_slot[t][j]] (in that order);
// u = RMSNorm(h) * gain.  blockDim = combine_threads(d): two float4 of the row
// per thread (so several CTAs share an SM and one wave covers the rows), the
// slots' loads issued four slots at a time.
__host__ __device__ constexpr int combine_threads(int d) { return ((d / 8 + 31) / 32) * 32; }

__global__ void __launch_bounds__(512) combine_norm_kernel(
    float* __restrict__ h, const float* __restrict__ yp, const int32_t* __restrict__ inv_slot,
    const float* __restrict__ gates, int k, int shared_base, int d, const uint16_t* __restrict__ gain, float eps,
    uint16_t* __restrict__ u, float* __restrict__ capture) {
  DG_TIMELINE_SCOPE(TLK_COMBINE_NORM);
  __shared__ float red[32];
  __shared__ int slot[ROW_MAX_K];
  __shared__ float gw[ROW_MAX_K];
  const int row = blockIdx.x, nv = d / 4;
  const int c0 = threadIdx.x, c1 = threadIdx.x + blockDim.x;
  const bool v0 = c0 < nv, v1 = c1 < nv;
  float4* hrow = reinterpret_cast<float4*>(h + static_cast<size_t>(row) * d);
  const float4* ys = reinterpret_cast<const float4*>(yp + static_cast<size_t>(shared_base + row) * d);
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 x0 = z, x1 = z, s0 = z, s1 = z;
  if (v0) {
    x0 = hrow[c0];
    s0 = ys[c0];
  }
  if (v1) {
    x1 = hrow[c1];
    s1 = ys[c1];
  }
  if (threadIdx.x < k) {
    slot[threadIdx.x] = inv_slot[static_cast<size_t>(row) * k + threadIdx.x];
    gw[threadIdx.x] = gates[static_cast<size_t>(row) * k + threadIdx.x];
  }
  __syncthreads();
  x0 = f4_add(x0, s0);
  x1 = f4_add(x1, s1);
  for (int q0 = 0; q0 < k; q0 += 4) {
    float4 y0[4], y1[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (q0 + q < k) {
        const float4* yr = reinterpret_cast<const float4*>(yp + static_cast<size_t>(slot[q0 + q]) * d);
        if (v0) y0[q] = yr[c0];
        if (v1) y1[q] = yr[c1];
      }
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (q0 + q < k) {
        if (v0) x0 = f4_fma(gw[q0 + q], y0[q], x0);
        if (v1) x1 = f4_fma(gw[q0 + q], y1[q], x1);
      }
  }
  float4 g0 = z, g1 = z;
  if (v0) {
    hrow[c0] = x0;
    if (capture) reinterpret_cast<float4*>(capture + static_cast<size_t>(row) * d)[c0] = x0;
    g0 = load_bf16x4(gain + 4 * c0);
  }
  if (v1) {
    hrow[c1] = x1;
    if (capture) reinterpret_cast<float4*>(capture + static_cast<size_t>(row) * d)[c1] = x1;
    g1 = load_bf16x4(gain + 4 * c1);
  }
  const float ss = block_sum((v0 ? f4_sumsq(x0) : 0.f) + (v1 ? f4_sumsq(x1) : 0.f), red);
  const float r = rsqrtf(ss / d + eps);
  uint16_t* urow = u + static_cast<size_t>(row) * d;
  if (v0) store_bf16x4(urow + 4 * c0, make_float4(x0.x * r * g0.x, x0.y * r * g0.y, x0.z * r * g0.z, x0.w * r * g0.w));
  if (v1) store_bf16x4(urow + 4 * c1, make_float4(x1.x * r * g1.x, x1.y * r * g1.y, x1.z * r * g1.z, x1.w * r * g1.w));
}

// Embedding gather (bf16 -> fp32 residual) + RMSNorm -> bf16.
// Token of row b*n+i: tokens[b * tok_stride + tok_off + i]; ids outside the
// vocabulary are clamped into it rather than read out of bounds.  add [rows, d]
// fp32 or NULL is added to the embedding (the self-conditioning signal).
__global__ void __launch_bounds__(1024) embed_norm_kernel(
    const int32_t* __restrict__ tokens, int tok_stride, int tok_off, int n, const uint16_t* __restrict__ embed,
    const uint16_t* __restrict__ gain, float eps, int d, float* __restrict__ h, uint16_t* __restrict__ u,
    float* __restrict__ capture, int32_t* settled, int n_settled, int vocab, const float* __restrict__ add) {
  DG_TIMELINE_SCOPE(TLK_EMBED_NORM);
  __shared__ float red[32];
  const int row = blockIdx.x, c = threadIdx.x;
  const int b = row / n, i = row % n;
  const bool valid = c < d / 4;
  if (settled != nullptr && row == 0 && threadIdx.x < n_settled) settled[threadIdx.x] = 1;
  const int tok = min(max(tokens[static_cast<size_t>(b) * tok_stride + tok_off + i], 0), vocab - 1);
  float4 x = make_float4(0.f, 0.f, 0.f, 0.f), g = x;
  if (valid) {
    g = load_bf16x4(gain + 4 * c);
    x = load_bf16x4(embed + static_cast<size_t>(tok) * d + 4 * c);
    if (add) x = f4_add(x, reinterpret_cast<const float4*>(add + static_cast<size_t>(row) * d)[c]);
    reinterpret_cast<float4*>(h + static_cast<size_t>(row) * d)[c] = x;
    if (capture) reinterpret_cast<float4*>(capture + static_cast<size_t>(row) * d)[c] = x;
  }
  norm_store_row(x, g, valid, d, eps, u + static_cast<size_t>(row) * d, red);
}

// h[row] += sum_s part[s][row] (splits in order); u[row] = RMSNorm(h[row]) * gain
__global__ void __launch_bounds__(1024) residual_norm_kernel(
    float* __restrict__ h, const float* __restrict__ part, int splits, int T, int d,
    const uint16_t* __restrict__ gain, float eps, uint16_t* __restrict__ u) {
  DG_TIMELINE_SCOPE(TLK_RESIDUAL_NORM);
  __shared__ float red[32];
  const int row = blockIdx.x, c = threadIdx.x;
  const bool valid = c < d / 4;
  float4* hrow = reinterpret_cast<float4*>(h + static_cast<size_t>(row) * d);
  float4 x = make_float4(0.f, 0.f, 0.f, 0.f), g = x;
  if (valid) {
    float4 pv[ROW_MAX_SPLITS];
    x = hrow[c];
    g = load_bf16x4(gain + 4 * c);
#pragma unroll
    for (int s = 0; s < ROW_MAX_SPLITS; ++s)
      if (s < splits) pv[s] = reinterpret_cast<const float4*>(part + (static_cast<size_t>(s) * T + row) * d)[c];
#pragma unroll
    for (int s = 0; s < ROW_MAX_SPLITS; ++s)
      if (s < splits) x = f4_add(x, pv[s]);
    hrow[c] = x;
  }
  norm_store_row(x, g, valid, d, eps, u + static_cast<size_t>(row) * d, red);
}

// Self-conditioning helpers (one CTA per row, one float4 per thread):
//   reduce_splits: out = sum_s part[s][row] (splits in order) as fp32 and / or bf16
//   swiglu_splits: out = SiLU(a[row]) * sum_s part[s][row], bf16 (a: the gate sums)
__global__ void __launch_bounds__(1024) reduce_splits_kernel(const float* __restrict__ part, int splits, int T,
                                                             int width, float* __restrict__ out_f32,
                                                             uint16_t* __restrict__ out_bf16) {
  DG_TIMELINE_SCOPE(TLK_REDUCE_SPLITS);
  const int row = blockIdx.x, c = threadIdx.x;
  if (c >= width / 4) return;
  float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < splits; s0 += 4) {
    float4 a[4];
#pragma unroll
    for (int s = 0; s < 4; ++s)
      if (s0 + s < splits) a[s] = reinterpret_cast<const float4*>(part + (static_cast<size_t>(s0 + s) * T + row) * width)[c];
#pragma unroll
    for (int s = 0; s < 4; ++s)
      if (s0 + s < splits) x = f4_add(x, a[s]);
  }
  if (out_f32) reinterpret_cast<float4*>(out_f32 + static_cast<size_t>(row) * width)[c] = x;
  if (out_bf16) store_bf16x4(out_bf16 + static_cast<size_t>(row) * width + 4 * c, x);
}

__global__ void __launch_bounds__(1024) swiglu_splits_kernel(const float* __restrict__ gate, const float* __restrict__ part,
                                                             int splits, int T, int width,
                                                             uint16_t* __restrict__ out_bf16) {
  DG_TIMELINE_SCOPE(TLK_SWIGLU_SPLITS);
  const int row = blockIdx.x, c = threadIdx.x;
  if (c >= width / 4) return;
  const float4 g = reinterpret_cast<const float4*>(gate + static_cast<size_t>(row) * width)[c];
  float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < splits; s0 += 4) {
    float4 a[4];
#pragma unroll
    for (int s = 0; s < 4; ++s)
      if (s0 + s < splits) a[s] = reinterpret_cast<const float4*>(part + (static_cast<size_t>(s0 + s) * T + row) * width)[c];
#pragma unroll
    for (int s = 0; s < 4; ++s)
      if (s0 + s < splits) x = f4_add(x, a[s]);
  }
  const auto silu = [](float v) { return v / (1.f + __expf(-v)); };
  store_bf16x4(out_bf16 + static_cast<size_t>(row) * width + 4 * c,
               make_float4(silu(g.x) * x.x, silu(g.y) * x.y, silu(g.z) * x.z, silu(g.w) * x.w));
}

// Reduce the QKV split-K partials (splits in order), rotate q and k pairs
// (j, j + D/2) at absolute position pos0 + i, write q [row][Hq][D] bf16 and
// k, v into this layer's cache [B][Hkv][S_max][D] at that position.  Four
// consecutive j per item (D/2 is a multiple of 4); blockIdx.y splits a row's
// items between CTAs, one item per thread.
__host__ __device__ constexpr int rope_items(int Hq, int Hkv, int D) { return (Hq + Hkv) * (D / 8) + Hkv * (D / 4); }
constexpr int ROPE_CTAS_PER_ROW = 2;
constexpr int ROPE_MAX_THREADS = 512;
constexpr int ROPE_BATCH = 3;  // split partials loaded per round trip (two CTAs of 512 threads per SM)

__global__ void __launch_bounds__(ROPE_MAX_THREADS, 2) rope_qkv_kernel(
    const float* __restrict__ part, int splits, int T, int n, int pos0, int Hq, int Hkv, int D,
    const float2* __restrict__ rope_tab, uint16_t* __restrict__ q, uint16_t* __restrict__ kc,
    uint16_t* __restrict__ vc, int S_max) {
  DG_TIMELINE_SCOPE(TLK_ROPE_QKV);
  const int row = blockIdx.x;
  const int b = row / n, i = row % n;
  const int pos = pos0 + i;
  const int QKV = (Hq + 2 * Hkv) * D;
  const int half = D / 2, hq4 = half / 4, d4 = D / 4;
  const float* base = part + static_cast<size_t>(row) * QKV;
  const size_t sstride = static_cast<size_t>(T) * QKV;
  const int n_rot = (Hq + Hkv) * hq4;
  for (int it = blockIdx.y * blockDim.x + threadIdx.x; it < n_rot + Hkv * d4; it += gridDim.y * blockDim.x) {
    if (it < n_rot) {
      const int hh = it / hq4, j = (it % hq4) * 4;
      const int c = hh * D + j;
      const float2* cs = rope_tab + static_cast<size_t>(pos) * half + j;
      const float2 c0 = cs[0], c1 = cs[1], c2 = cs[2], c3 = cs[3];
      float4 x1 = make_float4(0.f, 0.f, 0.f, 0.f), x2 = x1;
      // splits in batches of ROPE_BATCH, the batch's loads issued before its sums
      for (int s0 = 0; s0 < splits; s0 += ROPE_BATCH) {
        float4 a[ROPE_BATCH], bq[ROPE_BATCH];
#pragma unroll
        for (int s = 0; s < ROPE_BATCH; ++s)
          if (s0 + s < splits) {
            a[s] = *reinterpret_cast<const float4*>(base + (s0 + s) * sstride + c);
            bq[s] = *reinterpret_cast<const float4*>(base + (s0 + s) * sstride + c + half);
          }
#pragma unroll
        for (int s = 0; s < ROPE_BATCH; ++s)
          if (s0 + s < splits) {
            x1 = f4_add(x1, a[s]);
            x2 = f4_add(x2, bq[s]);
          }
      }
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
      for (int s0 = 0; s0 < splits; s0 += ROPE_BATCH) {
        float4 a[ROPE_BATCH];
#pragma unroll
        for (int s = 0; s < ROPE_BATCH; ++s)
          if (s0 + s < splits) a[s] = *reinterpret_cast<const float4*>(base + (s0 + s) * sstride + c);
#pragma unroll
        for (int s = 0; s < ROPE_BATCH; ++s)
          if (s0 + s < splits) x = f4_add(x, a[s]);
      }
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
  float s;   // sum 2^(x - m1)
  float s1;  // sum 2^(x - m1) * x
};

__device__ __forceinline__ Top2 top2_merge(Top2 a, Top2 b) {
  if (b.m1 == -INFINITY) return a;
  if (a.m1 == -INFINITY) return b;
  if (b.m1 > a.m1 || (b.m1 == a.m1 && b.idx < a.idx)) {
    const Top2 t = a;
    a = b;
    b = t;
  }
  const float sc = exp2f(b.m1 - a.m1);
  Top2 r;
  r.m1 = a.m1;
  r.idx = a.idx;
  r.m2 = fmaxf(a.m2, b.m1);
  r.s = a.s + b.s * sc;
  r.s1 = a.s1 + b.s1 * sc;
  return r;
}

// merge of one token's partials over the vocabulary tiles (one CTA per token)
__device__ __forceinline__ Top2 merge_token_partials(const float4* __restrict__ part, const float* __restrict__ s1,
                                                     int n_vtiles, int T, int t) {
  __shared__ Top2 sh[32];
  Top2 acc{-INFINITY, 0x7fffffff, -INFINITY, 0.f, 0.f};
  for (int v = threadIdx.x; v < n_vtiles; v += blockDim.x) {
    const float4 p = part[static_cast<size_t>(v) * T + t];
    acc = top2_merge(acc, Top2{p.x, __float_as_int(p.y), p.z, p.w, s1 ? s1[static_cast<size_t>(v) * T + t] : 0.f});
  }
  for (int o = 16; o > 0; o >>= 1) {
    Top2 other;
    other.m1 = __shfl_xor_sync(0xffffffffu, acc.m1, o);
    other.idx = __shfl_xor_sync(0xffffffffu, acc.idx, o);
    other.m2 = __shfl_xor_sync(0xffffffffu, acc.m2, o);
    other.s = __shfl_xor_sync(0xffffffffu, acc.s, o);
    other.s1 = __shfl_xor_sync(0xffffffffu, acc.s1, o);
    acc = top2_merge(acc, other);
  }
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0)
    for (int w = 1; w < (blockDim.x >> 5); ++w) acc = top2_merge(acc, sh[w]);
  return acc;  // valid in thread 0
}

// entropy of the softmax in nats from the merged statistics (log2 units):
// H = ln 2 * (m1 + log2 s - s1 / s)
__device__ __forceinline__ float merged_entropy(const Top2& a) {
  return (a.m1 + log2f(a.s) - a.s1 / a.s) * 0.69314718055994531f;
}

struct SampleArgs {
  int n_vtiles, T, C, P, step, vocab;
  uint32_t seed_lo, seed_hi;
  float tau;
  int stats_only;          // 1: write the statistics only (the entropy sampler decides)
  int32_t* canvas_out;
  float* conf_out;
  int32_t* settled;
  int32_t* dbg_argmax;
  float* dbg_lse;
  float* dbg_conf;
  float* dbg_margin;
  float* dbg_entropy;
  const float* s1;         // entropy partials [vocab tiles][T] or NULL
  float* lse2;             // log-sum-exp in log2 units [T] or NULL (self-conditioning)
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
  DG_TIMELINE_SCOPE(TLK_LMHEAD_MERGE_SAMPLE);
  const int t = blockIdx.x;
  const Top2 acc = merge_token_partials(part, a.s1, a.n_vtiles, a.T, t);
  if (threadIdx.x == 0) {
    const float conf = 1.f / acc.s;                      // exp(m1 - lse)
    const float lse = (acc.m1 + log2f(acc.s)) * 0.69314718055994531f;
    const float margin = (1.f - exp2f(acc.m2 - acc.m1)) / acc.s;
    const int b = t / a.C, i = t % a.C;
    if (!a.stats_only) {
      const int out = sample_decision(acc.idx, conf, a.tau, a.P + i, a.step, b, a.seed_lo, a.seed_hi, a.vocab);
      a.canvas_out[t] = out;
      if (a.conf_out) a.conf_out[t] = conf;
      if (a.settled && !(conf >= a.tau)) a.settled[b] = 0;
    }
    if (a.dbg_argmax) a.dbg_argmax[t] = acc.idx;
    if (a.dbg_lse) a.dbg_lse[t] = lse;
    if (a.dbg_conf) a.dbg_conf[t] = conf;
    if (a.dbg_margin) a.dbg_margin[t] = margin;
    if (a.dbg_entropy && a.s1) a.dbg_entropy[t] = merged_entropy(acc);
    if (a.lse2) a.lse2[t] = acc.m1 + log2f(acc.s);
  }
}

// Entropy-constrained sampler (codemajin.net "DiffusionGemma architecture",
// section 3.3), one CTA of C threads per sequence (C <= 256):
//   * adaptive stop when prev_argmax is given, the mean entropy of the canvas
//     is below stop_entropy and every argmax equals prev_argmax: every position
//     takes its argmax and stopped[b] = 1;
//   * otherwise positions in ascending (entropy, position) order are accepted
//     while the running sum of their entropies stays <= gamma (the first
//     always), the others take a uniform token (the same Philox draw as the
//     threshold sampler).
// The mean and the running sum are float32 sums taken in position order and
// in acceptance order by one thread, so a decision depends only on the
// float32 entropies.  argmax_out (may equal prev_argmax) receives the argmax.
struct EntropyArgs {
  int C, P, step, vocab;
  uint32_t seed_lo, seed_hi;
  float gamma, stop_entropy;
  const int32_t* argmax;      // [B*C] (merged statistics)
  const float* entropy;       // [B*C] nats
  const int32_t* prev_argmax; // [B*C] or NULL (first step of a block)
  int32_t* argmax_out;        // [B*C] or NULL
  int32_t* canvas_out;        // [B*C]
  float* entropy_out;         // [B*C] or NULL
  int32_t* stopped;           // [B] or NULL
};

__global__ void __launch_bounds__(256) entropy_sample_kernel(EntropyArgs a) {
  DG_TIMELINE_SCOPE(TLK_ENTROPY_SAMPLE);
  __shared__ float se[256];
  __shared__ int order[256];
  __shared__ int s_count;
  __shared__ int s_stop;
  const int b = blockIdx.x, i = threadIdx.x;
  const bool live = i < a.C;
  const size_t t = static_cast<size_t>(b) * a.C + i;
  const int am = live ? a.argmax[t] : 0;
  const float e = live ? a.entropy[t] : 0.f;
  const bool same = !live || (a.prev_argmax != nullptr && a.prev_argmax[t] == am);
  if (live) se[i] = e;
  const bool all_same = __syncthreads_and(same);
  // rank of (e, i) among the canvas: its place in the acceptance order
  if (live) {
    int rank = 0;
    for (int j = 0; j < a.C; ++j) rank += (se[j] < e || (se[j] == e && j < i)) ? 1 : 0;
    order[rank] = i;
  }
  __syncthreads();
  if (i == 0) {
    float sum = 0.f;
    for (int j = 0; j < a.C; ++j) sum += se[j];
    const float mean = sum / static_cast<float>(a.C);
    s_stop = (a.prev_argmax != nullptr && mean < a.stop_entropy && all_same) ? 1 : 0;
    float run = 0.f;
    int n = 0;
    for (int r = 0; r < a.C; ++r) {
      run += se[order[r]];
      if (r > 0 && !(run <= a.gamma)) break;
      ++n;
    }
    s_count = n;
  }
  __syncthreads();
  if (!live) return;
  int rank = 0;
  for (int j = 0; j < a.C; ++j) rank += (se[j] < e || (se[j] == e && j < i)) ? 1 : 0;
  int out = am;
  if (!s_stop && rank >= s_count) {
    const uint4 r = philox4x32_10(make_uint4(static_cast<uint32_t>(a.P + i), static_cast<uint32_t>(a.step),
                                             static_cast<uint32_t>(b), 0u),
                                  make_uint2(a.seed_lo, a.seed_hi));
    out = uniform_token(r.x, a.vocab);
  }
  a.canvas_out[t] = out;
  if (a.entropy_out) a.entropy_out[t] = e;
  if (a.argmax_out) a.argmax_out[t] = am;
  if (a.stopped && i == 0) a.stopped[b] = s_stop;
}

// sampler alone (test hook): given argmax / conf
__global__ void sample_only_kernel(const int32_t* __restrict__ argmax, const float* __restrict__ conf, int T,
                                   int C, int P, int step, uint32_t seed_lo, uint32_t seed_hi, float tau,
                                   int vocab, int32_t* __restrict__ out) {
  DG_TIMELINE_SCOPE(TLK_SAMPLE_ONLY);
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  out[t] = sample_decision(argmax[t], conf[t], tau, P + t % C, step, t / C, seed_lo, seed_hi, vocab);
}

// waits on a barrier that is never signalled; the bounded wait must give up
__global__ void wait_timeout_kernel(DevErr err) {
  DG_TIMELINE_SCOPE(TLK_OTHER);
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, err);
}

}  // namespace dg
