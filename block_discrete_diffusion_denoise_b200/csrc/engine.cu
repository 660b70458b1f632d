// C ABI of the denoising step (include/dg.h): context, workspace plan, TMA
// descriptors, the layer loop shared by the causal encoder (prefill, block
// commit) and the bidirectional decoder (denoising step), and test hooks.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/dg.h"
#include "attention_tc.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "kernels.cuh"

using namespace dg;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct LayerMaps {
  CUtensorMap wqkv, wo, wr, wg, wu, wd, wsg, wsu, wsd;
  CUtensorMap kc, vc;  // this layer's K / V cache rows, 64 x 64 boxes
};

// the sampler that ends a step
enum Sampler : int { SAMPLER_TAU = 0, SAMPLER_ENTROPY = 1, SAMPLER_COUNT = 2 };

// Step as one captured CUDA graph; a call rebinds the nodes whose arguments
// change: the embedding (canvas), the LM head (temperature) and the sampler.
struct StepGraph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  int B = -1, P = -1;
  cudaGraphNode_t embed_node = nullptr, sample_node = nullptr;
  std::vector<cudaGraphNode_t> lm_nodes;       // LM-head passes (statistics, then probabilities)
  cudaKernelNodeParams embed_kp{}, sample_kp{};
  std::vector<cudaKernelNodeParams> lm_kps;
  std::vector<void*> embed_args, sample_args;
  int64_t launches = 0;
  bool sc = false;                             // captured with self-conditioning
};

}  // namespace

struct dg_ctx {
  dg_config cfg{};
  int dev = 0;
  int sms = 148;
  cudaStream_t stream = nullptr;
  std::vector<dg_layer_weights> layers;
  const uint16_t* embed = nullptr;
  const uint16_t* final_norm = nullptr;
  const float* router_bias = nullptr;
  // sizes
  int d = 0, D = 0, Hq = 0, Hkv = 0, E = 0, k = 0, F = 0, Fs = 0, V = 0, L = 0, QKV = 0, HD = 0;
  int R = 0;        // workspace rows (max of step rows and prefill rows)
  int R_step = 0;   // max_batch * canvas
  size_t part_cap = 0;
  // device buffers
  void* ws = nullptr;
  uint16_t* kcache = nullptr;
  uint16_t* vcache = nullptr;
  float* h = nullptr;
  uint16_t* u = nullptr;
  float* part = nullptr;
  uint16_t* q = nullptr;
  uint16_t* o = nullptr;
  int32_t* idx = nullptr;
  float* gates = nullptr;
  int32_t* inv_slot = nullptr;     // routed row of each (token, slot) pair
  int32_t* chunk_done = nullptr;   // finished gate/up tiles per expert token chunk
  int32_t* expert_rows = nullptr;  // [E] rows routed to each expert (dispatch cursors)
  int32_t* moe_work = nullptr;     // claim / exit counters of the expert GEMM
  float* attn_part = nullptr;      // attention key-chunk partials: one 256-row slot per SM (sms x 272 rows x D)
  float2* attn_part_ml = nullptr;  // their row statistics: sms x 256 rows
  int32_t* dense_work = nullptr;   // claim / exit counters of the dense GEMM
  // CUDA graphs of the denoising step, one per sampler (per batch and cached length)
  bool use_graphs = true;
  StepGraph graphs[SAMPLER_COUNT];
  uint16_t* xp = nullptr;
  uint16_t* hbuf = nullptr;
  uint16_t* hsbuf = nullptr;
  float* yp = nullptr;
  float4* lm_part = nullptr;
  float2* rope = nullptr;
  int* err_word = nullptr;
  int32_t* dbg_argmax = nullptr;
  float* dbg_lse = nullptr;
  float* dbg_conf = nullptr;
  float* dbg_margin = nullptr;
  float* dbg_entropy = nullptr;
  float* lm_s1 = nullptr;          // LM-head entropy partials [V/128][R_step]
  // self-conditioning (weights optional): signal of the last step, added to
  // the next step's embeddings while sc_valid
  const uint16_t* sc_gate = nullptr;
  const uint16_t* sc_up = nullptr;
  const uint16_t* sc_down = nullptr;
  bool sc_enabled = false, sc_valid = false;
  bool capturing_graph = false;
  void* sc_ws = nullptr;
  uint16_t* sc_P = nullptr;        // [R_step][V] bf16 probabilities of the step
  float* sc_lse2 = nullptr;        // [R_step] log-sum-exp, log2 units
  uint16_t* sc_e = nullptr;        // [R_step][d] bf16 p . E
  float* sc_tmp = nullptr;         // [R_step][F] gate sums
  uint16_t* sc_h = nullptr;        // [R_step][F] bf16 SwiGLU hidden
  float* sc_sig = nullptr;         // [R_step][d] the signal
  CUtensorMap m_embed_mn{}, m_scP64{}, m_scP_store{}, m_sc_e64{}, m_sc_h64{}, m_sc_gate{}, m_sc_up{}, m_sc_down{};
  int32_t* io_canvas_in = nullptr;
  int32_t* io_canvas_out = nullptr;
  float* io_conf = nullptr;
  int32_t* io_settled = nullptr;
  size_t max_chunks = 0;
  // capture (test hook)
  bool capture = false;
  float* cap_h = nullptr;
  int32_t* cap_idx = nullptr;
  uint16_t* cap_u = nullptr;    // [L + 1][R_step][d]: router inputs per layer, then the LM-head input
  // tensor maps
  std::vector<LayerMaps> lmaps;
  CUtensorMap m_u16{}, m_u64{}, m_u128{}, m_o64{}, m_xp16{}, m_h16{}, m_hs16{}, m_embed{};
  CUtensorMap m_xp64{}, m_h64{}, m_hs64{};         // 64-row boxes (expert GEMM B)
  CUtensorMap m_q4{};  // queries as (D, G, Hkv, token): one GQA group's rows per box
  // state
  int B = 0;
  int P = 0;
  bool prefilled = false;
  uint64_t wait_limit_ns = 1000000000ull;
  bool trace = false;          // DG_TRACE=1: launch shapes to stderr
  int64_t launches = 0;
  std::string last_error;
  // profiling hook: event pairs per kernel class
  int prof_mask = 0;
  std::vector<cudaEvent_t> ev_pool;
  size_t ev_used = 0;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> prof_pairs[DG_PROF_CLASSES];
};

namespace {

dg_status fail(dg_ctx* c, dg_status s, const char* fmt, ...) {
  if (c) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    c->last_error = buf;
  }
  return s;
}

#define DG_CUDA(c, call)                                                                     \
  do {                                                                                       \
    cudaError_t e_ = (call);                                                                 \
    if (e_ != cudaSuccess) return fail((c), DG_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

#define DG_LAUNCHED(c)                                                                              \
  do {                                                                                              \
    (c)->launches++;                                                                                \
    cudaError_t e_ = cudaGetLastError();                                                            \
    if (e_ != cudaSuccess) return fail((c), DG_ERR_CUDA, "launch failed at %s:%d: %s", __FILE__, __LINE__, \
                                       cudaGetErrorString(e_));                                     \
  } while (0)

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

// bf16 matrix [rows, cols] row-major; box = 64 columns x box_rows rows, 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || base == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 split-K partials [splits][T][M] as 3-D (M, T, splits), box 128 x 64 x 1,
// no swizzle: the TMA-store epilogue of the dense GEMM (M a multiple of 4)
bool make_map_partials(CUtensorMap* m, void* base, int splits, int T, int M) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || base == nullptr || M % 4) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(splits)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(M) * 4, static_cast<cuuint64_t>(T) * M * 4};
  cuuint32_t box[3] = {128, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Queries [token][Hq][D] seen as 4-D (D, G, Hkv, token): a box of 64 columns x
// G heads x 1 kv head x 128/G tokens is the 128 packed rows (row = token * G +
// head) of one GQA group, 128-byte swizzled.  Requires 128 % G == 0.
bool make_map_q4(CUtensorMap* m, const void* base, uint64_t tokens, int Hkv, int G, int D) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || base == nullptr) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(G), static_cast<cuuint64_t>(Hkv), tokens};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(G) * D * 2,
                           static_cast<cuuint64_t>(Hkv) * G * D * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(G), 1, static_cast<cuuint32_t>(ATC_BQ / G)};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch on the context's stream (arguments converted to the kernel's types).
template <typename... KArgs, typename... Args>
cudaError_t launch(dg_ctx* c, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c->stream;
  cfg.numAttrs = 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

#define DG_LAUNCH(c, kern, grid, block, smem, ...)                                                           \
  do {                                                                                                      \
    const cudaError_t le_ = launch((c), kern, dim3(grid), dim3(block), (smem), __VA_ARGS__);               \
    if (le_ != cudaSuccess) return fail((c), DG_ERR_CUDA, "launch %s: %s", #kern, cudaGetErrorString(le_)); \
    DG_LAUNCHED(c);                                                                                         \
  } while (0)

DevErr dev_err(const dg_ctx* c) { return DevErr{c->err_word, c->wait_limit_ns}; }

// Profiling hook: an event pair around the launches of one kernel class.
struct ProfScope {
  dg_ctx* c;
  int cls;
  cudaEvent_t stop = nullptr;
  ProfScope(dg_ctx* ctx, int k) : c(ctx), cls(k) {
    if (!(c->prof_mask >> cls & 1)) return;
    if (c->ev_used + 2 > c->ev_pool.size()) {
      for (int i = 0; i < 64; ++i) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return;
        c->ev_pool.push_back(e);
      }
    }
    cudaEvent_t start = c->ev_pool[c->ev_used++];
    stop = c->ev_pool[c->ev_used++];
    cudaEventRecord(start, c->stream);
    c->prof_pairs[cls].push_back({start, stop});
  }
  void end() {
    if (stop) cudaEventRecord(stop, c->stream);
    stop = nullptr;
  }
  ~ProfScope() { end(); }
};

// out[s][t][m] = partial sums over split s of W[m, :] . X[t, :]
// x: token rows with 64-row TMA boxes
dg_status gemm_dense(dg_ctx* c, const CUtensorMap& w, const CUtensorMap& x, int M, int T, int K, int* splits_out,
                     int max_splits = 11, bool a_mn_major = false) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.a_map[0] = w;
  p.a_mn_major = a_mn_major ? 1 : 0;
  p.b_map = x;
  p.b_box_rows = 64;
  p.M = M;
  p.T = T;
  p.k_steps = K / 64;
  const int m_tiles = (M + GEMM_BM - 1) / GEMM_BM;
  const size_t cap_s = c->part_cap / (static_cast<size_t>(T) * M);
  // Token-tile width and split count from a per-CTA cost model fitted to
  // in-kernel phase stamps of these GEMMs on B200 (µs): ~2.3 to the first
  // operands, 0.12 + 0.28*bn/256 per 64-wide k-step, 4.4*bn/256 for the
  // epilogue, plus ~0.3 per split for the consumer that sums the partials.
  const int widths[3] = {std::min(DENSE_BN, (T + 15) / 16 * 16), 128, 64};
  double best = 1e30;
  int best_bn = widths[0], best_s = 1;
  for (int wi = 0; wi < 3; ++wi) {
    const int bnc = widths[wi];
    if (wi > 0 && bnc >= widths[0]) continue;
    const int nt = (T + bnc - 1) / bnc;
    for (int sp = 1; sp <= 8; ++sp) {
      if (p.k_steps / sp < 4 || static_cast<size_t>(sp) > std::min<size_t>({cap_s, static_cast<size_t>(max_splits),
                                                                             static_cast<size_t>(ROW_MAX_SPLITS)}))
        break;
      const int ctas = m_tiles * nt * sp;
      const double rounds = std::ceil(static_cast<double>(ctas) / c->sms);
      const double per_cta = 2.3 + (static_cast<double>(p.k_steps) / sp) * (0.12 + 0.28 * bnc / 256.0) +
                             4.4 * bnc / 256.0;
      const double cost = rounds * per_cta + 0.3 * sp;
      if (cost < best - 1e-9) {
        best = cost;
        best_bn = bnc;
        best_s = sp;
      }
    }
  }
  p.bn = best_bn;
  p.n_tiles_n = (T + p.bn - 1) / p.bn;
  p.splits = best_s;
  p.tiles_static = m_tiles * p.n_tiles_n * p.splits;
  p.out_f32 = c->part;
  p.use_tma_store = make_map_partials(&p.out_map, c->part, p.splits, T, M) ? 1 : 0;
  p.work = c->dense_work;
  p.err = dev_err(c);
  ProfScope ps0(c, DG_PROF_DENSE);
  DG_LAUNCH(c, gemm_kernel<GEMM_DENSE>, std::min(c->sms, p.tiles_static), GEMM_THREADS,
            gemm_smem_bytes<GEMM_DENSE>(), p);
  ps0.end();
  *splits_out = p.splits;
  return DG_OK;
}

dg_status attention(dg_ctx* c, int l, int B, int n, int pos0, bool causal) {
  AttnTcParams p;
  p.q_map = c->m_q4;
  p.k_map = c->lmaps[l].kc;
  p.v_map = c->lmaps[l].vc;
  p.o = c->o;
  p.part = c->attn_part;
  p.part_ml = c->attn_part_ml;
  p.n = n;
  p.B = B;
  p.Hq = c->Hq;
  p.Hkv = c->Hkv;
  p.S_max = c->cfg.max_seq;
  p.pos0 = pos0;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c->D)));
  p.err = dev_err(c);
  const int G = c->Hq / c->Hkv;
  const int qblocks = (n * G + ATC_ROWS - 1) / ATC_ROWS;
  const int units = qblocks * B * c->Hkv;
  const int keys = pos0 + n;
  // Split the keys into chunks so that units x chunks fills the SMs in one
  // wave (the partial buffer holds one slot per SM), at least four 64-key
  // blocks per chunk; several chunks are combined by attn_merge_kernel.
  int n_chunks = std::max(1, std::min({ATC_MAX_CHUNKS, c->sms / std::max(1, units), keys / (4 * ATC_BK)}));
  const int chunk_len = ((keys + n_chunks - 1) / n_chunks + ATC_BK - 1) / ATC_BK * ATC_BK;
  n_chunks = (keys + chunk_len - 1) / chunk_len;
  p.chunk_len = chunk_len;
  p.n_chunks = n_chunks;
  if (c->trace && l == 0)
    fprintf(stderr, "[dg] attention: keys %d, units %d, chunks %d x %d keys\n", keys, units, n_chunks, chunk_len);
  const dim3 grid(qblocks, B * c->Hkv, n_chunks);
  const dim3 mgrid(units, (ATC_ROWS * (c->D / 4) + 255) / 256);
  const float4* part4 = reinterpret_cast<const float4*>(c->attn_part);
  ProfScope ps1(c, DG_PROF_ATTENTION);
  switch (c->D) {
    case 64:
      DG_LAUNCH(c, attn_tc_kernel<64>, grid, ATC_THREADS, AtcCfg<64>::SMEM, p);
      if (n_chunks > 1)
        DG_LAUNCH(c, attn_merge_kernel<64>, mgrid, 256, 0, part4, static_cast<const float2*>(c->attn_part_ml),
                  n_chunks, qblocks, n, c->Hq, c->Hkv, c->o);
      break;
    case 128:
      DG_LAUNCH(c, attn_tc_kernel<128>, grid, ATC_THREADS, AtcCfg<128>::SMEM, p);
      if (n_chunks > 1)
        DG_LAUNCH(c, attn_merge_kernel<128>, mgrid, 256, 0, part4, static_cast<const float2*>(c->attn_part_ml),
                  n_chunks, qblocks, n, c->Hq, c->Hkv, c->o);
      break;
    case 176:
      DG_LAUNCH(c, attn_tc_kernel<176>, grid, ATC_THREADS, AtcCfg<176>::SMEM, p);
      if (n_chunks > 1)
        DG_LAUNCH(c, attn_merge_kernel<176>, mgrid, 256, 0, part4, static_cast<const float2*>(c->attn_part_ml),
                  n_chunks, qblocks, n, c->Hq, c->Hkv, c->o);
      break;
    default:
      return fail(c, DG_ERR_UNSUPPORTED, "head_dim %d", c->D);
  }
  ps1.end();
  return DG_OK;
}

// record: capture the expert choices (denoising steps only: the capture
// buffers hold R_step rows per layer)
dg_status moe(dg_ctx* c, int l, int T, bool record) {
  const LayerMaps& lm = c->lmaps[l];
  int s3 = 1;
  dg_status st = gemm_dense(c, lm.wr, c->m_u64, c->E, T, c->d, &s3);
  if (st != DG_OK) return st;
  int32_t* cap = (record && c->capture) ? c->cap_idx + static_cast<size_t>(l) * c->R_step * c->k : nullptr;
  // routing: the top-k decision of every token with the claim of its rows in
  // the experts' regions and the copy of its activations (one warp per token)
  ProfScope ps3(c, DG_PROF_ROUTING);
  // expert e's rows: [e * T, e * T + rows_e) (a region per expert, T rows each)
  // two tokens (warps) per CTA: the k copies of every token's row spread over many SMs
  auto* dispatch = c->E <= 32 ? route_dispatch_kernel<1>
                   : c->E <= 64 ? route_dispatch_kernel<2>
                   : c->E <= 128 ? route_dispatch_kernel<4> : route_dispatch_kernel<ROUTE_PER>;
  DG_LAUNCH(c, dispatch, T, 32 * c->k, 0, static_cast<const float*>(c->part), s3, T, c->E, c->k,
            c->router_bias, c->idx, c->gates, cap, c->expert_rows, T, c->d, static_cast<const uint16_t*>(c->u),
            c->xp, c->inv_slot);
  ps3.end();

  // routed + shared experts, gate/up then down, one persistent launch
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.a_map[0] = lm.wg;
  p.a_map[1] = lm.wu;
  p.as_map[0] = lm.wsg;
  p.as_map[1] = lm.wsu;
  p.b_map = c->m_xp16;
  p.bs_map = c->m_u16;
  p.d_map = lm.wd;
  p.ds_map = lm.wsd;
  p.h_map = c->m_h16;
  p.hs_map = c->m_hs16;
  p.b_mid_map = c->m_xp64;
  p.bs_mid_map = c->m_u64;
  p.h_mid_map = c->m_h64;
  p.hs_mid_map = c->m_hs64;
  p.b_mid_rows = 64;
  p.b_box_rows = 16;
  p.T = T;
  p.expert_rows = c->expert_rows;
  p.region = T;
  p.work = c->moe_work;
  p.chunk_done = c->chunk_done;
  p.n_groups_routed = c->E;
  p.F = c->F;
  p.Fs = c->Fs;
  p.d = c->d;
  p.h_out = c->hbuf;
  p.hs_out = c->hsbuf;
  p.out_f32 = c->yp;
  p.out_ld = c->d;
  p.shared_row_base = c->E * T;
  p.err = dev_err(c);
  ProfScope ps6(c, DG_PROF_EXPERTS);
  DG_LAUNCH(c, gemm_kernel<GEMM_MOE>, c->sms, GEMM_THREADS, gemm_smem_bytes<GEMM_MOE>(), p);
  ps6.end();
  return DG_OK;
}

// Forward of B x n new rows at positions [pos0, pos0 + n).
//   causal = true : encoder (prefill chunk / block commit); K/V are written
//                   to the cache; the last layer stops after its K/V.
//   causal = false: denoising step; canvas K/V go to cache rows [P, P+C)
//                   (beyond the committed length), then the LM head runs.
dg_status forward(dg_ctx* c, const int32_t* tokens, int tok_stride, int tok_off, int B, int n, int pos0,
                  bool causal, int32_t* settled) {
  const int T = B * n;
  const float eps = c->cfg.rms_eps;
  float* cap0 = (c->capture && !causal) ? c->cap_h : nullptr;
  ProfScope ps8(c, DG_PROF_OTHER);
  const float* sc_add = (!causal && c->sc_enabled && (c->sc_valid || c->capturing_graph)) ? c->sc_sig : nullptr;
  DG_LAUNCH(c, embed_norm_kernel, T, row_threads(c->d), 0, tokens, tok_stride, tok_off, n, c->embed,
            static_cast<const uint16_t*>(c->layers[0].attn_norm), eps, c->d, c->h, c->u, cap0, settled, B, c->V,
            sc_add);
  ps8.end();
  for (int l = 0; l < c->L; ++l) {
    const LayerMaps& lm = c->lmaps[l];
    const dg_layer_weights& lw = c->layers[l];
    int s1 = 1;
    dg_status st = gemm_dense(c, lm.wqkv, c->m_u64, c->QKV, T, c->d, &s1);
    if (st != DG_OK) return st;
    const size_t layer_off = static_cast<size_t>(l) * c->cfg.max_batch * c->Hkv * c->cfg.max_seq * c->D;
    ProfScope ps9(c, DG_PROF_OTHER);
    DG_LAUNCH(c, rope_qkv_kernel, dim3(T, ROPE_CTAS_PER_ROW),
              std::min(ROPE_MAX_THREADS,
                       (rope_items(c->Hq, c->Hkv, c->D) + ROPE_CTAS_PER_ROW * 32 - 1) / (ROPE_CTAS_PER_ROW * 32) * 32),
              0,
              static_cast<const float*>(c->part), s1, T, n, pos0, c->Hq, c->Hkv,
              c->D, static_cast<const float2*>(c->rope), c->q, c->kcache + layer_off, c->vcache + layer_off,
              c->cfg.max_seq);
    ps9.end();
    if (causal && l == c->L - 1) break;  // only this layer's keys/values feed the cache
    st = attention(c, l, B, n, pos0, causal);
    if (st != DG_OK) return st;
    int s2 = 1;
    st = gemm_dense(c, lm.wo, c->m_o64, c->d, T, c->HD, &s2);
    if (st != DG_OK) return st;
    ProfScope ps10(c, DG_PROF_OTHER);
    DG_LAUNCH(c, residual_norm_kernel, T, row_threads(c->d), 0, c->h, static_cast<const float*>(c->part), s2, T, c->d,
              static_cast<const uint16_t*>(lw.ffn_norm), eps, c->u);
    ps10.end();
    if (c->capture && !causal)
      DG_CUDA(c, cudaMemcpyAsync(c->cap_u + static_cast<size_t>(l) * c->R_step * c->d, c->u,
                                 static_cast<size_t>(T) * c->d * 2, cudaMemcpyDeviceToDevice, c->stream));
    st = moe(c, l, T, !causal);
    if (st != DG_OK) return st;
    const uint16_t* next_gain = l + 1 < c->L ? static_cast<const uint16_t*>(c->layers[l + 1].attn_norm)
                                             : c->final_norm;
    float* cap = (c->capture && !causal) ? c->cap_h + static_cast<size_t>(l + 1) * c->R_step * c->d : nullptr;
    ProfScope ps11(c, DG_PROF_OTHER);
    DG_LAUNCH(c, combine_norm_kernel, T, combine_threads(c->d), 0, c->h, static_cast<const float*>(c->yp),
              static_cast<const int32_t*>(c->inv_slot), static_cast<const float*>(c->gates), c->k, c->E * T,
              c->d, next_gain, eps, c->u, cap);
    ps11.end();
    if (c->capture && !causal && l == c->L - 1)
      DG_CUDA(c, cudaMemcpyAsync(c->cap_u + static_cast<size_t>(c->L) * c->R_step * c->d, c->u,
                                 static_cast<size_t>(T) * c->d * 2, cudaMemcpyDeviceToDevice, c->stream));
  }
  return DG_OK;
}

// LM head over the B*C canvas rows with the per-(vocabulary tile, row)
// statistics, at the given temperature
dg_status lm_head(dg_ctx* c, int T, float temperature) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.a_map[0] = c->m_u128;
  p.b_map = c->m_embed;
  p.b_box_rows = 128;
  p.M = T;
  p.k_steps = c->d / 64;
  p.n_mtiles = (T + GEMM_BM - 1) / GEMM_BM;
  p.tiles_static = (c->V / GEMM_BN) * lmhead_mpairs(p.n_mtiles);
  p.lm_part = c->lm_part;
  p.lm_s1 = c->lm_s1;
  p.logit_scale_log2 = static_cast<float>(1.4426950408889634 / static_cast<double>(temperature));
  p.err = dev_err(c);
  ProfScope ps12(c, DG_PROF_LMHEAD);
  DG_LAUNCH(c, gemm_kernel<GEMM_LMHEAD>, std::min(c->sms, p.tiles_static), GEMM_THREADS,
            gemm_smem_bytes<GEMM_LMHEAD>(), p);
  ps12.end();
  return DG_OK;
}

SampleArgs merge_args(const dg_ctx* c, int T, bool stats_only) {
  SampleArgs a;
  memset(&a, 0, sizeof(a));
  a.n_vtiles = c->V / GEMM_BN;
  a.T = T;
  a.C = c->cfg.canvas;
  a.P = c->P;
  a.vocab = c->V;
  a.stats_only = stats_only ? 1 : 0;
  a.dbg_argmax = c->dbg_argmax;
  a.dbg_lse = c->dbg_lse;
  a.dbg_conf = c->dbg_conf;
  a.dbg_margin = c->dbg_margin;
  a.dbg_entropy = c->dbg_entropy;
  a.s1 = c->lm_s1;
  a.lse2 = c->sc_enabled ? c->sc_lse2 : nullptr;
  return a;
}

// Self-conditioning signal of this step (codemajin.net "DiffusionGemma
// architecture", section 3.2): p = softmax(z E^T / T) written as bf16 by a
// second LM-head pass (the statistics pass gave the log-sum-exp), e = p E by
// a split-K GEMM with E as an MN-major A operand, then the SwiGLU feed-forward
// layer; the next step adds the result to its embeddings.
dg_status self_condition(dg_ctx* c, int T, float temperature) {
  {
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.a_map[0] = c->m_u128;
    p.b_map = c->m_embed;
    p.b_box_rows = 128;
    p.M = T;
    p.k_steps = c->d / 64;
    p.n_mtiles = (T + GEMM_BM - 1) / GEMM_BM;
    p.tiles_static = (c->V / GEMM_BN) * lmhead_mpairs(p.n_mtiles);
    p.lse2 = c->sc_lse2;
    p.p_map = c->m_scP_store;
    p.logit_scale_log2 = static_cast<float>(1.4426950408889634 / static_cast<double>(temperature));
    p.err = dev_err(c);
    ProfScope ps(c, DG_PROF_LMHEAD);
    DG_LAUNCH(c, gemm_kernel<GEMM_LMHEAD>, std::min(c->sms, p.tiles_static), GEMM_THREADS,
              gemm_smem_bytes<GEMM_LMHEAD>(), p);
    ps.end();
  }
  int s = 1;
  dg_status st = gemm_dense(c, c->m_embed_mn, c->m_scP64, c->d, T, c->V, &s, 8, true);
  if (st != DG_OK) return st;
  ProfScope ps(c, DG_PROF_OTHER);
  DG_LAUNCH(c, reduce_splits_kernel, T, row_threads(c->d), 0, static_cast<const float*>(c->part), s, T, c->d,
            static_cast<float*>(nullptr), c->sc_e);
  ps.end();
  st = gemm_dense(c, c->m_sc_gate, c->m_sc_e64, c->F, T, c->d, &s);
  if (st != DG_OK) return st;
  ProfScope ps2(c, DG_PROF_OTHER);
  DG_LAUNCH(c, reduce_splits_kernel, T, row_threads(c->F), 0, static_cast<const float*>(c->part), s, T, c->F,
            c->sc_tmp, static_cast<uint16_t*>(nullptr));
  ps2.end();
  st = gemm_dense(c, c->m_sc_up, c->m_sc_e64, c->F, T, c->d, &s);
  if (st != DG_OK) return st;
  ProfScope ps3(c, DG_PROF_OTHER);
  DG_LAUNCH(c, swiglu_splits_kernel, T, row_threads(c->F), 0, static_cast<const float*>(c->sc_tmp),
            static_cast<const float*>(c->part), s, T, c->F, c->sc_h);
  ps3.end();
  st = gemm_dense(c, c->m_sc_down, c->m_sc_h64, c->d, T, c->F, &s);
  if (st != DG_OK) return st;
  ProfScope ps4(c, DG_PROF_OTHER);
  DG_LAUNCH(c, reduce_splits_kernel, T, row_threads(c->d), 0, static_cast<const float*>(c->part), s, T, c->d,
            c->sc_sig, static_cast<uint16_t*>(nullptr));
  ps4.end();
  return DG_OK;
}

// threshold sampler: merge of the LM-head statistics + Philox re-noising
dg_status lm_head_and_sample(dg_ctx* c, int B, int step, uint64_t seed, float tau, int32_t* canvas_out,
                             float* conf_out, int32_t* settled) {
  const int T = B * c->cfg.canvas;
  dg_status st = lm_head(c, T, c->cfg.temperature);
  if (st != DG_OK) return st;
  SampleArgs a = merge_args(c, T, false);
  a.step = step;
  a.seed_lo = static_cast<uint32_t>(seed & 0xFFFFFFFFull);
  a.seed_hi = static_cast<uint32_t>(seed >> 32);
  a.tau = tau;
  a.canvas_out = canvas_out;
  a.conf_out = conf_out;
  a.settled = settled;
  ProfScope ps13(c, DG_PROF_OTHER);
  DG_LAUNCH(c, lmhead_merge_sample_kernel, T, 256, 0, static_cast<const float4*>(c->lm_part), a);
  ps13.end();
  if (c->sc_enabled) return self_condition(c, T, c->cfg.temperature);
  return DG_OK;
}

struct EntropyCall {
  int step;
  uint64_t seed;
  dg_entropy_args args;
  const int32_t* prev_argmax;
  int32_t* argmax_out;
  int32_t* canvas_out;
  float* entropy_out;
  int32_t* stopped;
};

EntropyArgs entropy_args(const dg_ctx* c, const EntropyCall& e) {
  EntropyArgs a;
  memset(&a, 0, sizeof(a));
  a.C = c->cfg.canvas;
  a.P = c->P;
  a.step = e.step;
  a.vocab = c->V;
  a.seed_lo = static_cast<uint32_t>(e.seed & 0xFFFFFFFFull);
  a.seed_hi = static_cast<uint32_t>(e.seed >> 32);
  a.gamma = e.args.gamma;
  a.stop_entropy = e.args.stop_entropy;
  a.argmax = c->dbg_argmax;
  a.entropy = c->dbg_entropy;
  a.prev_argmax = e.prev_argmax;
  a.argmax_out = e.argmax_out;
  a.canvas_out = e.canvas_out;
  a.entropy_out = e.entropy_out;
  a.stopped = e.stopped;
  return a;
}

// entropy-constrained sampler: LM head at this step's temperature, merged
// statistics, then the per-sequence ordering / budget / stop rule
dg_status lm_head_and_entropy_sample(dg_ctx* c, int B, const EntropyCall& e) {
  const int T = B * c->cfg.canvas;
  dg_status st = lm_head(c, T, e.args.temperature);
  if (st != DG_OK) return st;
  SampleArgs a = merge_args(c, T, true);
  ProfScope ps13(c, DG_PROF_OTHER);
  DG_LAUNCH(c, lmhead_merge_sample_kernel, T, 256, 0, static_cast<const float4*>(c->lm_part), a);
  DG_LAUNCH(c, entropy_sample_kernel, B, 256, 0, entropy_args(c, e));
  ps13.end();
  if (c->sc_enabled) return self_condition(c, T, e.args.temperature);
  return DG_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

template <typename T>
T* carve(char*& cur, size_t count) {
  T* p = reinterpret_cast<T*>(cur);
  cur += (count * sizeof(T) + 255) / 256 * 256;
  return p;
}

// rows of one forward (tokens of a step or of a prefill chunk): the expert
// GEMM's tile tables count rows and chunks in 16 bits
constexpr int kMaxRows = 32768;
static_assert(PERM_MAXE == MOE_MAX_EXPERTS, "routing and expert GEMM agree on the expert limit");

// every kernel's dynamic shared memory fits the 227 KB a CTA may opt into
constexpr int kMaxSmemPerCta = 232448;
static_assert(gemm_smem_bytes<GEMM_DENSE>() <= kMaxSmemPerCta, "dense GEMM shared memory");
static_assert(gemm_smem_bytes<GEMM_MOE>() <= kMaxSmemPerCta, "expert GEMM shared memory");
static_assert(gemm_smem_bytes<GEMM_LMHEAD>() <= kMaxSmemPerCta, "LM-head GEMM shared memory");
static_assert(AtcCfg<64>::SMEM <= kMaxSmemPerCta && AtcCfg<128>::SMEM <= kMaxSmemPerCta &&
                  AtcCfg<176>::SMEM <= kMaxSmemPerCta,
              "attention shared memory");

dg_status set_smem_attrs(dg_ctx* c) {
  DG_CUDA(c, cudaFuncSetAttribute(gemm_kernel<GEMM_DENSE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  gemm_smem_bytes<GEMM_DENSE>()));
  DG_CUDA(c, cudaFuncSetAttribute(gemm_kernel<GEMM_MOE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  gemm_smem_bytes<GEMM_MOE>()));
  DG_CUDA(c, cudaFuncSetAttribute(gemm_kernel<GEMM_LMHEAD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  gemm_smem_bytes<GEMM_LMHEAD>()));
  DG_CUDA(c, cudaFuncSetAttribute(attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, AtcCfg<64>::SMEM));
  DG_CUDA(c, cudaFuncSetAttribute(attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, AtcCfg<128>::SMEM));
  DG_CUDA(c, cudaFuncSetAttribute(attn_tc_kernel<176>, cudaFuncAttributeMaxDynamicSharedMemorySize, AtcCfg<176>::SMEM));
  return DG_OK;
}

void drop_step_graph(StepGraph& g) {
  if (g.exec) cudaGraphExecDestroy(g.exec);
  if (g.graph) cudaGraphDestroy(g.graph);
  g = StepGraph();
}

void drop_step_graphs(dg_ctx* c) {
  for (StepGraph& g : c->graphs) drop_step_graph(g);
}

// Capture the whole step (embedding .. sampler) with the given sampler once
// per (batch, cached length) on the context stream.
dg_status capture_step(dg_ctx* c, int mode) {
  StepGraph& sg = c->graphs[mode];
  drop_step_graph(sg);
  const int64_t l0 = c->launches;
  DG_CUDA(c, cudaStreamBeginCapture(c->stream, cudaStreamCaptureModeThreadLocal));
  c->capturing_graph = true;
  dg_status st = forward(c, c->io_canvas_in, c->cfg.canvas, 0, c->B, c->cfg.canvas, c->P, false,
                         mode == SAMPLER_TAU ? c->io_settled : nullptr);
  if (st == DG_OK) {
    if (mode == SAMPLER_TAU) {
      st = lm_head_and_sample(c, c->B, 0, 0, 0.f, c->io_canvas_out, c->io_conf, c->io_settled);
    } else {
      EntropyCall e{};
      e.args.temperature = 1.f;
      e.canvas_out = c->io_canvas_out;
      st = lm_head_and_entropy_sample(c, c->B, e);
    }
  }
  c->capturing_graph = false;
  cudaGraph_t g = nullptr;
  const cudaError_t ce = cudaStreamEndCapture(c->stream, &g);
  if (st != DG_OK || ce != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    cudaGetLastError();
    return st != DG_OK ? st : fail(c, DG_ERR_CUDA, "step capture: %s", cudaGetErrorString(ce));
  }
  sg.graph = g;
  DG_CUDA(c, cudaGraphInstantiate(&sg.exec, g, 0));
  size_t n = 0;
  DG_CUDA(c, cudaGraphGetNodes(g, nullptr, &n));
  std::vector<cudaGraphNode_t> nodes(n);
  DG_CUDA(c, cudaGraphGetNodes(g, nodes.data(), &n));
  const void* sampler_fn = mode == SAMPLER_TAU ? reinterpret_cast<const void*>(lmhead_merge_sample_kernel)
                                               : reinterpret_cast<const void*>(entropy_sample_kernel);
  for (cudaGraphNode_t nd : nodes) {
    cudaGraphNodeType ty;
    if (cudaGraphNodeGetType(nd, &ty) != cudaSuccess || ty != cudaGraphNodeTypeKernel) continue;
    cudaKernelNodeParams kp;
    if (cudaGraphKernelNodeGetParams(nd, &kp) != cudaSuccess) continue;
    if (kp.func == reinterpret_cast<void*>(embed_norm_kernel)) {
      sg.embed_node = nd;
      sg.embed_kp = kp;
    } else if (kp.func == reinterpret_cast<void*>(gemm_kernel<GEMM_LMHEAD>)) {
      sg.lm_nodes.push_back(nd);
      sg.lm_kps.push_back(kp);
    } else if (kp.func == sampler_fn) {
      sg.sample_node = nd;
      sg.sample_kp = kp;
    }
  }
  if (!sg.embed_node || sg.lm_nodes.empty() || !sg.sample_node) {
    drop_step_graph(sg);
    return fail(c, DG_ERR_CUDA, "step graph: entry/exit kernels not found");
  }
  // argument pointer arrays: point at the graph's stored values except the rebound ones
  sg.embed_args.assign(sg.embed_kp.kernelParams, sg.embed_kp.kernelParams + 15);
  sg.sample_args.assign(sg.sample_kp.kernelParams, sg.sample_kp.kernelParams + (mode == SAMPLER_TAU ? 2 : 1));
  sg.launches = c->launches - l0;
  c->launches = l0;
  sg.B = c->B;
  sg.P = c->P;
  sg.sc = c->sc_enabled;
  return DG_OK;
}

// rebind the embedding node: canvas and settled flags
dg_status rebind_embed(dg_ctx* c, StepGraph& sg, const int32_t* canvas_in, int32_t* settled) {
  // embed_norm_kernel(tokens, tok_stride, tok_off, n, embed, gain, eps, d, h, u, capture, settled, n_settled, vocab)
  const int32_t* tok = canvas_in;
  int32_t* set0 = settled;
  const float* add = (c->sc_enabled && c->sc_valid) ? c->sc_sig : nullptr;
  std::vector<void*> ea = sg.embed_args;
  ea[0] = &tok;
  ea[11] = &set0;
  ea[14] = &add;
  cudaKernelNodeParams ekp = sg.embed_kp;
  ekp.kernelParams = ea.data();
  DG_CUDA(c, cudaGraphExecKernelNodeSetParams(sg.exec, sg.embed_node, &ekp));
  return DG_OK;
}

dg_status launch_graph(dg_ctx* c, StepGraph& sg) {
  DG_CUDA(c, cudaGraphLaunch(sg.exec, c->stream));
  c->launches += sg.launches;
  return DG_OK;
}

// threshold sampler step as a graph: rebinds the first kernel (canvas,
// settled flags) and the last one (step, seed, tau, outputs)
dg_status step_via_graph(dg_ctx* c, const int32_t* canvas_in, int32_t step, uint64_t seed, float tau,
                         int32_t* canvas_out, float* conf, int32_t* settled) {
  StepGraph& sg = c->graphs[SAMPLER_TAU];
  if (!sg.exec || sg.B != c->B || sg.P != c->P || sg.sc != c->sc_enabled) {
    dg_status st = capture_step(c, SAMPLER_TAU);
    if (st != DG_OK) return st;
  }
  dg_status st = rebind_embed(c, sg, canvas_in, settled);
  if (st != DG_OK) return st;
  // lmhead_merge_sample_kernel(part, SampleArgs)
  SampleArgs a = *static_cast<SampleArgs*>(sg.sample_args[1]);
  a.step = step;
  a.seed_lo = static_cast<uint32_t>(seed & 0xFFFFFFFFull);
  a.seed_hi = static_cast<uint32_t>(seed >> 32);
  a.tau = tau;
  a.canvas_out = canvas_out;
  a.conf_out = conf;
  a.settled = settled;
  std::vector<void*> sa = sg.sample_args;
  sa[1] = &a;
  cudaKernelNodeParams skp = sg.sample_kp;
  skp.kernelParams = sa.data();
  DG_CUDA(c, cudaGraphExecKernelNodeSetParams(sg.exec, sg.sample_node, &skp));
  return launch_graph(c, sg);
}

// entropy sampler step as a graph: rebinds the embedding (canvas), the LM
// head (temperature) and the entropy sampler (its arguments)
dg_status entropy_step_via_graph(dg_ctx* c, const int32_t* canvas_in, const EntropyCall& e) {
  StepGraph& sg = c->graphs[SAMPLER_ENTROPY];
  if (!sg.exec || sg.B != c->B || sg.P != c->P || sg.sc != c->sc_enabled) {
    dg_status st = capture_step(c, SAMPLER_ENTROPY);
    if (st != DG_OK) return st;
  }
  dg_status st = rebind_embed(c, sg, canvas_in, nullptr);
  if (st != DG_OK) return st;
  for (size_t i = 0; i < sg.lm_nodes.size(); ++i) {
    GemmParams lp = *static_cast<GemmParams*>(sg.lm_kps[i].kernelParams[0]);
    lp.logit_scale_log2 = static_cast<float>(1.4426950408889634 / static_cast<double>(e.args.temperature));
    void* la[1] = {&lp};
    cudaKernelNodeParams lkp = sg.lm_kps[i];
    lkp.kernelParams = la;
    DG_CUDA(c, cudaGraphExecKernelNodeSetParams(sg.exec, sg.lm_nodes[i], &lkp));
  }
  EntropyArgs ea = entropy_args(c, e);
  void* sa[1] = {&ea};
  cudaKernelNodeParams skp = sg.sample_kp;
  skp.kernelParams = sa;
  DG_CUDA(c, cudaGraphExecKernelNodeSetParams(sg.exec, sg.sample_node, &skp));
  return launch_graph(c, sg);
}

void free_all(dg_ctx* c) {
  drop_step_graphs(c);
  for (cudaEvent_t e : c->ev_pool) cudaEventDestroy(e);
  c->ev_pool.clear();
  if (c->ws) cudaFree(c->ws);
  if (c->kcache) cudaFree(c->kcache);
  if (c->vcache) cudaFree(c->vcache);
  if (c->cap_h) cudaFree(c->cap_h);
  if (c->cap_idx) cudaFree(c->cap_idx);
  if (c->cap_u) cudaFree(c->cap_u);
  if (c->sc_ws) cudaFree(c->sc_ws);
  c->sc_ws = nullptr;
  c->ws = nullptr;
  c->kcache = c->vcache = nullptr;
  c->cap_h = nullptr;
  c->cap_idx = nullptr;
  c->cap_u = nullptr;
}

}  // namespace

// =============================================================================
// C ABI
// =============================================================================
namespace {

// The calling thread's last dg_create failure (a failed create has no
// context to carry it); dg_last_error(NULL) returns it.
thread_local std::string g_create_error;

// free a context that dg_create gives up on, keeping its message
void discard(dg_ctx* c) {
  g_create_error = "dg_create: " + c->last_error;
  delete c;
}

}  // namespace

extern "C" {

dg_status dg_create(const dg_config* cfg, const dg_weights* w, void* cuda_stream, dg_ctx** out) {
  if (!cfg || !w || !out) {
    g_create_error = "dg_create: null argument";
    return DG_ERR_INVALID_ARG;
  }
  g_create_error.clear();
  *out = nullptr;
  dg_ctx* c = new dg_ctx();
  c->cfg = *cfg;
  dg_config& g = c->cfg;
  if (g.prefill_rows <= 0) g.prefill_rows = 2048;
  auto reject = [&](dg_status s, const char* why) {
    g_create_error = std::string("dg_create: ") + why;
    delete c;
    return s;
  };
  if (g.n_layers <= 0 || g.d_model <= 0 || g.n_q_heads <= 0 || g.n_kv_heads <= 0 || g.n_experts <= 0 ||
      g.top_k <= 0 || g.expert_hidden <= 0 || g.shared_hidden <= 0 || g.vocab <= 0 || g.canvas <= 0 ||
      g.max_batch <= 0 || g.max_seq <= 0 || !(g.rms_eps >= 0.f) || !(g.temperature > 0.f) ||
      !(g.rope_base > 0.f))
    return reject(DG_ERR_INVALID_ARG, "non-positive dimension");
  if (g.d_model % 128 || g.d_model > 4096 || g.expert_hidden % 64 || g.shared_hidden % 64 || g.vocab % 128 ||
      (g.head_dim != 64 && g.head_dim != 128 && g.head_dim != 176) || g.n_q_heads % g.n_kv_heads ||
      (g.n_q_heads * g.head_dim) % 64 || ATC_BQ % (g.n_q_heads / g.n_kv_heads) || g.n_experts > PERM_MAXE || g.n_experts % 4 || g.top_k > 16 || g.top_k > g.n_experts ||
      g.canvas % 16 || g.canvas > 256 || g.max_seq < g.canvas)
    return reject(DG_ERR_UNSUPPORTED, "unsupported shape");
  if (!w->embed || !w->final_norm || !w->layers) return reject(DG_ERR_INVALID_ARG, "null weights");
  c->layers.assign(w->layers, w->layers + g.n_layers);
  for (const auto& lw : c->layers) {
    const void* ptrs[] = {lw.attn_norm, lw.wqkv, lw.wo, lw.ffn_norm, lw.w_router, lw.w_gate,
                          lw.w_up, lw.w_down, lw.ws_gate, lw.ws_up, lw.ws_down};
    for (const void* pp : ptrs)
      if (!pp || !aligned16(pp)) return reject(DG_ERR_INVALID_ARG, "layer weight null or not 16-byte aligned");
  }
  if (!aligned16(w->embed)) return reject(DG_ERR_INVALID_ARG, "embed not 16-byte aligned");
  c->embed = static_cast<const uint16_t*>(w->embed);
  c->final_norm = static_cast<const uint16_t*>(w->final_norm);
  if (w->sc_gate || w->sc_up || w->sc_down) {
    if (!w->sc_gate || !w->sc_up || !w->sc_down || !aligned16(w->sc_gate) || !aligned16(w->sc_up) ||
        !aligned16(w->sc_down))
      return reject(DG_ERR_INVALID_ARG, "self-conditioning weights: all three, 16-byte aligned");
    c->sc_gate = static_cast<const uint16_t*>(w->sc_gate);
    c->sc_up = static_cast<const uint16_t*>(w->sc_up);
    c->sc_down = static_cast<const uint16_t*>(w->sc_down);
  }
  c->router_bias = w->router_bias;
  c->stream = static_cast<cudaStream_t>(cuda_stream);
  c->d = g.d_model;
  c->D = g.head_dim;
  c->Hq = g.n_q_heads;
  c->Hkv = g.n_kv_heads;
  c->E = g.n_experts;
  c->k = g.top_k;
  c->F = g.expert_hidden;
  c->Fs = g.shared_hidden;
  c->V = g.vocab;
  c->L = g.n_layers;
  c->QKV = (c->Hq + 2 * c->Hkv) * c->D;
  c->HD = c->Hq * c->D;
  c->R_step = g.max_batch * g.canvas;
  c->R = std::max(c->R_step, g.prefill_rows);
  if (c->R > kMaxRows) return reject(DG_ERR_UNSUPPORTED, "max_batch * canvas and prefill_rows must be <= 32768");
  if (const char* s = getenv("DG_WAIT_LIMIT_NS")) c->wait_limit_ns = strtoull(s, nullptr, 10);
  if (const char* s = getenv("DG_TRACE")) c->trace = atoi(s) != 0;

  cudaError_t e = cudaGetDevice(&c->dev);
  if (e != cudaSuccess) {
    dg_status st = fail(c, DG_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    discard(c);
    return st;
  }
  cudaDeviceGetAttribute(&c->sms, cudaDevAttrMultiProcessorCount, c->dev);
  if (set_smem_attrs(c) != DG_OK) {
    discard(c);
    return DG_ERR_CUDA;
  }


  // ---- workspace plan ----
  const size_t R = c->R, d = c->d, k = c->k;
  const size_t mmax = std::max<size_t>({static_cast<size_t>(c->QKV), d, static_cast<size_t>(c->E)});
  c->part_cap = std::max<size_t>(R, 5 * 256) * mmax;
  const size_t CH = MOE_CHUNK_ROWS;
  const size_t chunks_max = (R * k + CH - 1) / CH + c->E;  // routed token chunks
  const size_t chunks_shared = (R + CH - 1) / CH;
  c->max_chunks = chunks_max + chunks_shared;
  // routed rows: expert e owns rows [e * T, e * T + rows_e) of xp, hbuf and yp
  // for a forward of T <= R rows (shared-expert outputs follow at E * T)
  const size_t ER = static_cast<size_t>(c->E) * R;
  size_t bytes = 0;
  auto add = [&](size_t n, size_t sz) { bytes += (n * sz + 255) / 256 * 256; };
  add(R * d, 4);                                  // h
  add(R * d, 2);                                  // u
  add(c->part_cap, 4);                            // part
  add(R * c->HD, 2);                              // q
  add(R * c->HD, 2);                              // o
  add(R * k, 4);                                  // idx
  add(R * k, 4);                                  // gates
  add(R * k, 4);                                  // inv_slot
  add(c->max_chunks, 4);                          // chunk_done
  add(PERM_MAXE, 4);                              // expert_rows
  add(2, 4);                                      // moe_work
  add(static_cast<size_t>(c->sms) * (ATC_ROWS + ATC_MAX_CHUNKS) * c->D, 4);  // attn_part
  add(static_cast<size_t>(c->sms) * ATC_ROWS, 8);         // attn_part_ml
  add(2, 4);                                      // dense_work
  add(ER * d, 2);                                 // xp
  add(ER * c->F, 2);                              // hbuf
  add(R * c->Fs, 2);                              // hsbuf
  add((ER + R) * d, 4);                           // yp
  add(static_cast<size_t>(c->V / GEMM_BN) * c->R_step, 16);  // lm_part
  add(static_cast<size_t>(c->V / GEMM_BN) * c->R_step, 4);   // lm_s1
  add(static_cast<size_t>(g.max_seq) * (c->D / 2), 8);        // rope
  add(4, 4);                                      // err word
  add(c->R_step, 4);                              // dbg_argmax
  add(c->R_step, 4);
  add(c->R_step, 4);
  add(c->R_step, 4);
  add(c->R_step, 4);                              // dbg_entropy
  add(c->R_step, 4);                              // io canvas in
  add(c->R_step, 4);                              // io canvas out
  add(c->R_step, 4);                              // io conf
  add(g.max_batch, 4);                            // io settled
  e = cudaMalloc(&c->ws, bytes);
  if (e != cudaSuccess) {
    dg_status st = fail(c, DG_ERR_OOM, "workspace %zu bytes: %s", bytes, cudaGetErrorString(e));
    discard(c);
    return st;
  }
  char* cur = static_cast<char*>(c->ws);
  c->h = carve<float>(cur, R * d);
  c->u = carve<uint16_t>(cur, R * d);
  c->part = carve<float>(cur, c->part_cap);
  c->q = carve<uint16_t>(cur, R * c->HD);
  c->o = carve<uint16_t>(cur, R * c->HD);
  c->idx = carve<int32_t>(cur, R * k);
  c->gates = carve<float>(cur, R * k);
  c->inv_slot = carve<int32_t>(cur, R * k);
  c->chunk_done = carve<int32_t>(cur, c->max_chunks);
  c->expert_rows = carve<int32_t>(cur, PERM_MAXE);
  c->moe_work = carve<int32_t>(cur, 2);
  c->attn_part = carve<float>(cur, static_cast<size_t>(c->sms) * (ATC_ROWS + ATC_MAX_CHUNKS) * c->D);
  c->attn_part_ml = carve<float2>(cur, static_cast<size_t>(c->sms) * ATC_ROWS);
  c->dense_work = carve<int32_t>(cur, 2);
  c->xp = carve<uint16_t>(cur, ER * d);
  c->hbuf = carve<uint16_t>(cur, ER * c->F);
  c->hsbuf = carve<uint16_t>(cur, R * c->Fs);
  c->yp = carve<float>(cur, (ER + R) * d);
  c->lm_part = carve<float4>(cur, static_cast<size_t>(c->V / GEMM_BN) * c->R_step);
  c->lm_s1 = carve<float>(cur, static_cast<size_t>(c->V / GEMM_BN) * c->R_step);
  c->rope = carve<float2>(cur, static_cast<size_t>(g.max_seq) * (c->D / 2));
  c->err_word = carve<int>(cur, 4);
  c->dbg_argmax = carve<int32_t>(cur, c->R_step);
  c->dbg_lse = carve<float>(cur, c->R_step);
  c->dbg_conf = carve<float>(cur, c->R_step);
  c->dbg_margin = carve<float>(cur, c->R_step);
  c->dbg_entropy = carve<float>(cur, c->R_step);
  c->io_canvas_in = carve<int32_t>(cur, c->R_step);
  c->io_canvas_out = carve<int32_t>(cur, c->R_step);
  c->io_conf = carve<float>(cur, c->R_step);
  c->io_settled = carve<int32_t>(cur, g.max_batch);

  const size_t cache_elems = static_cast<size_t>(c->L) * g.max_batch * c->Hkv * g.max_seq * c->D;
  e = cudaMalloc(&c->kcache, cache_elems * 2);
  if (e == cudaSuccess) e = cudaMalloc(&c->vcache, cache_elems * 2);
  if (e != cudaSuccess) {
    dg_status st = fail(c, DG_ERR_OOM, "KV cache 2 x %zu bytes: %s", cache_elems * 2, cudaGetErrorString(e));
    free_all(c);
    discard(c);
    return st;
  }
  // zero everything once: stale rows of token-side operands then hold finite values
  cudaMemsetAsync(c->ws, 0, bytes, c->stream);
  cudaMemsetAsync(c->kcache, 0, cache_elems * 2, c->stream);
  cudaMemsetAsync(c->vcache, 0, cache_elems * 2, c->stream);

  // RoPE table: angle pos * base^(-2j/D) in double precision, stored fp32
  {
    const int half = c->D / 2;
    std::vector<float2> tab(static_cast<size_t>(g.max_seq) * half);
    for (int pos = 0; pos < g.max_seq; ++pos)
      for (int j = 0; j < half; ++j) {
        const double inv = std::pow(static_cast<double>(g.rope_base), -2.0 * j / c->D);
        const double a = pos * inv;
        tab[static_cast<size_t>(pos) * half + j] = make_float2(static_cast<float>(std::cos(a)),
                                                               static_cast<float>(std::sin(a)));
      }
    e = cudaMemcpyAsync(c->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice, c->stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(c->stream);
    if (e != cudaSuccess) {
      dg_status st = fail(c, DG_ERR_CUDA, "rope upload: %s", cudaGetErrorString(e));
      free_all(c);
      discard(c);
      return st;
    }
  }

  // ---- TMA descriptors ----
  bool ok = true;
  c->lmaps.resize(c->L);
  for (int l = 0; l < c->L; ++l) {
    const dg_layer_weights& lw = c->layers[l];
    LayerMaps& m = c->lmaps[l];
    ok &= make_map(&m.wqkv, lw.wqkv, c->QKV, d, 128);
    ok &= make_map(&m.wo, lw.wo, d, c->HD, 128);
    ok &= make_map(&m.wr, lw.w_router, c->E, d, 128);
    ok &= make_map(&m.wg, lw.w_gate, static_cast<uint64_t>(c->E) * c->F, d, 64);
    ok &= make_map(&m.wu, lw.w_up, static_cast<uint64_t>(c->E) * c->F, d, 64);
    ok &= make_map(&m.wd, lw.w_down, static_cast<uint64_t>(c->E) * d, c->F, 128);
    ok &= make_map(&m.wsg, lw.ws_gate, c->Fs, d, 64);
    ok &= make_map(&m.wsu, lw.ws_up, c->Fs, d, 64);
    ok &= make_map(&m.wsd, lw.ws_down, d, c->Fs, 128);
    const size_t layer_off = static_cast<size_t>(l) * g.max_batch * c->Hkv * g.max_seq * c->D;
    const uint64_t cache_rows = static_cast<uint64_t>(g.max_batch) * c->Hkv * g.max_seq;
    ok &= make_map(&m.kc, c->kcache + layer_off, cache_rows, c->D, 64);
    ok &= make_map(&m.vc, c->vcache + layer_off, cache_rows, c->D, 64);
  }
  ok &= make_map_q4(&c->m_q4, c->q, R, c->Hkv, c->Hq / c->Hkv, c->D);
  ok &= make_map(&c->m_u16, c->u, R, d, 16);
  ok &= make_map(&c->m_u64, c->u, R, d, 64);
  ok &= make_map(&c->m_u128, c->u, R, d, 128);
  ok &= make_map(&c->m_o64, c->o, R, c->HD, 64);
  ok &= make_map(&c->m_xp16, c->xp, ER, d, 16);
  ok &= make_map(&c->m_xp64, c->xp, ER, d, 64);
  ok &= make_map(&c->m_h64, c->hbuf, ER, c->F, 64);
  ok &= make_map(&c->m_hs64, c->hsbuf, R, c->Fs, 64);
  ok &= make_map(&c->m_h16, c->hbuf, ER, c->F, 16);
  ok &= make_map(&c->m_hs16, c->hsbuf, R, c->Fs, 16);
  ok &= make_map(&c->m_embed, c->embed, c->V, d, 128);
  if (ok && c->sc_gate) {
    const size_t RS = c->R_step, V = c->V, F = c->F;
    const size_t sc_bytes = ((RS * V * 2 + 255) / 256 + (RS * 4 + 255) / 256 + (RS * d * 2 + 255) / 256 +
                             (RS * F * 4 + 255) / 256 + (RS * F * 2 + 255) / 256 + (RS * d * 4 + 255) / 256) * 256;
    if (cudaMalloc(&c->sc_ws, sc_bytes) != cudaSuccess) {
      dg_status st = fail(c, DG_ERR_OOM, "self-conditioning buffers %zu bytes", sc_bytes);
      free_all(c);
      discard(c);
      return st;
    }
    cudaMemsetAsync(c->sc_ws, 0, sc_bytes, c->stream);
    char* sc = static_cast<char*>(c->sc_ws);
    c->sc_P = carve<uint16_t>(sc, RS * V);
    c->sc_lse2 = carve<float>(sc, RS);
    c->sc_e = carve<uint16_t>(sc, RS * d);
    c->sc_tmp = carve<float>(sc, RS * F);
    c->sc_h = carve<uint16_t>(sc, RS * F);
    c->sc_sig = carve<float>(sc, RS * d);
    ok &= make_map(&c->m_embed_mn, c->embed, c->V, d, 64);      // E as [V][d]: A of p . E, MN-major
    ok &= make_map(&c->m_scP64, c->sc_P, RS, V, 64);             // p as the B operand
    ok &= make_map(&c->m_scP_store, c->sc_P, RS, V, 128);        // p stored by the LM-head pass
    ok &= make_map(&c->m_sc_e64, c->sc_e, RS, d, 64);
    ok &= make_map(&c->m_sc_h64, c->sc_h, RS, F, 64);
    ok &= make_map(&c->m_sc_gate, c->sc_gate, F, d, 128);
    ok &= make_map(&c->m_sc_up, c->sc_up, F, d, 128);
    ok &= make_map(&c->m_sc_down, c->sc_down, d, F, 128);
  }
  if (!ok) {
    dg_status st = fail(c, DG_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    free_all(c);
    discard(c);
    return st;
  }
  *out = c;
  return DG_OK;
}

dg_status dg_destroy(dg_ctx* c) {
  if (!c) return DG_ERR_INVALID_ARG;
  cudaStreamSynchronize(c->stream);
  free_all(c);
  delete c;
  return DG_OK;
}

dg_status dg_prefill(dg_ctx* c, const int32_t* tokens, int32_t B, int32_t P) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (!tokens || B <= 0 || P <= 0) return fail(c, DG_ERR_INVALID_ARG, "prefill: bad arguments");
  if (B > c->cfg.max_batch || P + c->cfg.canvas > c->cfg.max_seq)
    return fail(c, DG_ERR_CAPACITY, "prefill: batch %d / length %d beyond capacity", B, P);
  c->B = B;
  c->P = 0;
  c->prefilled = false;
  c->sc_valid = false;  // a new canvas starts without a self-conditioning signal
  const int chunk = std::max(1, c->R / B);
  for (int p0 = 0; p0 < P; p0 += chunk) {
    const int n = std::min(chunk, P - p0);
    dg_status st = forward(c, tokens, P, p0, B, n, p0, true, nullptr);
    if (st != DG_OK) return st;
  }
  c->P = P;
  c->prefilled = true;
  return DG_OK;
}

dg_status dg_denoise_step(dg_ctx* c, const int32_t* canvas_in, int32_t step, uint64_t seed, float tau,
                          int32_t* canvas_out, float* conf, int32_t* settled) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (!canvas_in || !canvas_out || !conf) return fail(c, DG_ERR_INVALID_ARG, "step: null buffer");
  if (!c->prefilled) return fail(c, DG_ERR_STATE, "step before prefill");
  if (c->P + c->cfg.canvas > c->cfg.max_seq) return fail(c, DG_ERR_CAPACITY, "step: cache full");
  dg_status st;
  // test hooks (capture, profiling) need the eager launches
  if (c->use_graphs && !c->capture && c->prof_mask == 0 && c->stream != nullptr) {
    st = step_via_graph(c, canvas_in, step, seed, tau, canvas_out, conf, settled);
  } else {
    st = forward(c, canvas_in, c->cfg.canvas, 0, c->B, c->cfg.canvas, c->P, false, settled);
    if (st == DG_OK) st = lm_head_and_sample(c, c->B, step, seed, tau, canvas_out, conf, settled);
  }
  if (st == DG_OK && c->sc_enabled) c->sc_valid = true;
  return st;
}

dg_status dg_denoise_step_entropy(dg_ctx* c, const int32_t* canvas_in, int32_t step, uint64_t seed,
                                  const dg_entropy_args* args, const int32_t* prev_argmax, int32_t* argmax_out,
                                  int32_t* canvas_out, float* entropy, int32_t* stopped) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (!canvas_in || !canvas_out || !args) return fail(c, DG_ERR_INVALID_ARG, "step_entropy: null argument");
  if (!(args->temperature > 0.f) || !(args->gamma >= 0.f) || args->stop_entropy != args->stop_entropy)
    return fail(c, DG_ERR_INVALID_ARG, "step_entropy: temperature must be > 0, gamma >= 0");
  if (!c->prefilled) return fail(c, DG_ERR_STATE, "step before prefill");
  if (c->P + c->cfg.canvas > c->cfg.max_seq) return fail(c, DG_ERR_CAPACITY, "step: cache full");
  EntropyCall e{step, seed, *args, prev_argmax, argmax_out, canvas_out, entropy, stopped};
  dg_status st;
  if (c->use_graphs && !c->capture && c->prof_mask == 0 && c->stream != nullptr) {
    st = entropy_step_via_graph(c, canvas_in, e);
  } else {
    st = forward(c, canvas_in, c->cfg.canvas, 0, c->B, c->cfg.canvas, c->P, false, nullptr);
    if (st == DG_OK) st = lm_head_and_entropy_sample(c, c->B, e);
  }
  if (st == DG_OK && c->sc_enabled) c->sc_valid = true;
  return st;
}

dg_status dg_denoise_step_host(dg_ctx* c, const int32_t* canvas_in_host, int32_t step, uint64_t seed, float tau,
                               int32_t* canvas_out_host, float* conf_host, int32_t* settled_host) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (!canvas_in_host || !canvas_out_host) return fail(c, DG_ERR_INVALID_ARG, "step_host: null buffer");
  if (!c->prefilled) return fail(c, DG_ERR_STATE, "step before prefill");
  const size_t T = static_cast<size_t>(c->B) * c->cfg.canvas;
  DG_CUDA(c, cudaMemcpyAsync(c->io_canvas_in, canvas_in_host, T * 4, cudaMemcpyHostToDevice, c->stream));
  dg_status st = dg_denoise_step(c, c->io_canvas_in, step, seed, tau, c->io_canvas_out, c->io_conf,
                                 settled_host ? c->io_settled : nullptr);
  if (st != DG_OK) return st;
  DG_CUDA(c, cudaMemcpyAsync(canvas_out_host, c->io_canvas_out, T * 4, cudaMemcpyDeviceToHost, c->stream));
  if (conf_host) DG_CUDA(c, cudaMemcpyAsync(conf_host, c->io_conf, T * 4, cudaMemcpyDeviceToHost, c->stream));
  if (settled_host)
    DG_CUDA(c, cudaMemcpyAsync(settled_host, c->io_settled, c->B * 4, cudaMemcpyDeviceToHost, c->stream));
  return dg_sync(c);
}

dg_status dg_commit_block(dg_ctx* c, const int32_t* block) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (!block) return fail(c, DG_ERR_INVALID_ARG, "commit: null block");
  if (!c->prefilled) return fail(c, DG_ERR_STATE, "commit before prefill");
  if (c->P + 2 * c->cfg.canvas > c->cfg.max_seq)
    return fail(c, DG_ERR_CAPACITY, "commit: no room for another block");
  dg_status st = forward(c, block, c->cfg.canvas, 0, c->B, c->cfg.canvas, c->P, true, nullptr);
  if (st != DG_OK) return st;
  c->P += c->cfg.canvas;
  c->sc_valid = false;  // the next block starts without a self-conditioning signal
  return DG_OK;
}

dg_status dg_sync(dg_ctx* c) {
  if (!c) return DG_ERR_INVALID_ARG;
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  int word = 0;
  DG_CUDA(c, cudaMemcpy(&word, c->err_word, 4, cudaMemcpyDeviceToHost));
  if (word != 0) {
    DG_CUDA(c, cudaMemset(c->err_word, 0, 4));
    return fail(c, DG_ERR_DEVICE_TIMEOUT, "a device wait exceeded %llu ns (code %d)",
                static_cast<unsigned long long>(c->wait_limit_ns), word);
  }
  return DG_OK;
}

int32_t dg_cached_len(const dg_ctx* c) { return c ? c->P : -1; }

const char* dg_last_error(const dg_ctx* c) {
  if (c) return c->last_error.c_str();
  return g_create_error.empty() ? "null context" : g_create_error.c_str();
}

dg_status dg_debug_capture(dg_ctx* c, int32_t enable) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (enable && !c->cap_h) {
    DG_CUDA(c, cudaMalloc(&c->cap_h, static_cast<size_t>(c->L + 1) * c->R_step * c->d * 4));
    DG_CUDA(c, cudaMalloc(&c->cap_idx, static_cast<size_t>(c->L) * c->R_step * c->k * 4));
    DG_CUDA(c, cudaMalloc(&c->cap_u, static_cast<size_t>(c->L + 1) * c->R_step * c->d * 2));
  }
  if (!enable && c->cap_h) {
    cudaStreamSynchronize(c->stream);
    cudaFree(c->cap_h);
    cudaFree(c->cap_idx);
    cudaFree(c->cap_u);
    c->cap_h = nullptr;
    c->cap_idx = nullptr;
    c->cap_u = nullptr;
  }
  c->capture = enable != 0;
  return DG_OK;
}

dg_status dg_debug_hidden(dg_ctx* c, int32_t layer, float* out) {
  if (!c || !out || !c->cap_h || layer < 0 || layer > c->L) return fail(c, DG_ERR_INVALID_ARG, "debug_hidden");
  const size_t n = static_cast<size_t>(c->B) * c->cfg.canvas * c->d;
  DG_CUDA(c, cudaMemcpyAsync(out, c->cap_h + static_cast<size_t>(layer) * c->R_step * c->d, n * 4,
                             cudaMemcpyDeviceToDevice, c->stream));
  return DG_OK;
}

dg_status dg_debug_experts(dg_ctx* c, int32_t layer, int32_t* out) {
  if (!c || !out || !c->cap_idx || layer < 0 || layer >= c->L) return fail(c, DG_ERR_INVALID_ARG, "debug_experts");
  const size_t n = static_cast<size_t>(c->B) * c->cfg.canvas * c->k;
  DG_CUDA(c, cudaMemcpyAsync(out, c->cap_idx + static_cast<size_t>(layer) * c->R_step * c->k, n * 4,
                             cudaMemcpyDeviceToDevice, c->stream));
  return DG_OK;
}

dg_status dg_debug_norm_rows(dg_ctx* c, int32_t layer, void* out) {
  if (!c || !out || !c->cap_u || layer < 0 || layer > c->L) return fail(c, DG_ERR_INVALID_ARG, "debug_norm_rows");
  const size_t n = static_cast<size_t>(c->B) * c->cfg.canvas * c->d;
  DG_CUDA(c, cudaMemcpyAsync(out, c->cap_u + static_cast<size_t>(layer) * c->R_step * c->d, n * 2,
                             cudaMemcpyDeviceToDevice, c->stream));
  return DG_OK;
}

dg_status dg_debug_lmhead(dg_ctx* c, int32_t* argmax, float* lse, float* conf, float* margin) {
  if (!c) return DG_ERR_INVALID_ARG;
  const size_t n = static_cast<size_t>(c->B) * c->cfg.canvas;
  if (argmax) DG_CUDA(c, cudaMemcpyAsync(argmax, c->dbg_argmax, n * 4, cudaMemcpyDeviceToDevice, c->stream));
  if (lse) DG_CUDA(c, cudaMemcpyAsync(lse, c->dbg_lse, n * 4, cudaMemcpyDeviceToDevice, c->stream));
  if (conf) DG_CUDA(c, cudaMemcpyAsync(conf, c->dbg_conf, n * 4, cudaMemcpyDeviceToDevice, c->stream));
  if (margin) DG_CUDA(c, cudaMemcpyAsync(margin, c->dbg_margin, n * 4, cudaMemcpyDeviceToDevice, c->stream));
  return DG_OK;
}

dg_status dg_debug_router(dg_ctx* c, const float* logits, int32_t n_rows, int32_t* idx, float* gates) {
  if (!c || !logits || !idx || !gates || n_rows <= 0) return fail(c, DG_ERR_INVALID_ARG, "debug_router");
  router_topk_kernel<<<n_rows, 256, 0, c->stream>>>(logits, 1, n_rows, c->E, c->k, nullptr, idx, gates);
  DG_LAUNCHED(c);
  return DG_OK;
}

dg_status dg_debug_sample(dg_ctx* c, const int32_t* argmax, const float* conf, int32_t B, int32_t step,
                          uint64_t seed, float tau, int32_t* out) {
  if (!c || !argmax || !conf || !out || B <= 0) return fail(c, DG_ERR_INVALID_ARG, "debug_sample");
  const int T = B * c->cfg.canvas;
  sample_only_kernel<<<(T + 255) / 256, 256, 0, c->stream>>>(argmax, conf, T, c->cfg.canvas, c->P, step,
                                                              static_cast<uint32_t>(seed & 0xFFFFFFFFull),
                                                              static_cast<uint32_t>(seed >> 32), tau, c->V, out);
  DG_LAUNCHED(c);
  return DG_OK;
}

dg_status dg_debug_entropy_sample(dg_ctx* c, const int32_t* argmax, const float* entropy, const int32_t* prev,
                                  int32_t B, int32_t step, uint64_t seed, float gamma, float stop_entropy,
                                  int32_t* out, int32_t* stopped) {
  if (!c || !argmax || !entropy || !out || B <= 0 || B > c->cfg.max_batch)
    return fail(c, DG_ERR_INVALID_ARG, "debug_entropy_sample");
  EntropyArgs a;
  memset(&a, 0, sizeof(a));
  a.C = c->cfg.canvas;
  a.P = c->P;
  a.step = step;
  a.vocab = c->V;
  a.seed_lo = static_cast<uint32_t>(seed & 0xFFFFFFFFull);
  a.seed_hi = static_cast<uint32_t>(seed >> 32);
  a.gamma = gamma;
  a.stop_entropy = stop_entropy;
  a.argmax = argmax;
  a.entropy = entropy;
  a.prev_argmax = prev;
  a.canvas_out = out;
  a.stopped = stopped;
  entropy_sample_kernel<<<B, 256, 0, c->stream>>>(a);
  DG_LAUNCHED(c);
  return DG_OK;
}

dg_status dg_set_self_conditioning(dg_ctx* c, int32_t enable) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (enable && !c->sc_ws) return fail(c, DG_ERR_UNSUPPORTED, "self-conditioning needs sc_gate/sc_up/sc_down");
  c->sc_enabled = enable != 0;
  c->sc_valid = false;
  return DG_OK;
}

dg_status dg_debug_self_cond(dg_ctx* c, float* out) {
  if (!c || !out || !c->sc_ws) return fail(c, DG_ERR_INVALID_ARG, "debug_self_cond");
  DG_CUDA(c, cudaMemcpyAsync(out, c->sc_sig, static_cast<size_t>(c->B) * c->cfg.canvas * c->d * 4,
                             cudaMemcpyDeviceToDevice, c->stream));
  return DG_OK;
}

dg_status dg_debug_entropy(dg_ctx* c, float* out) {
  if (!c || !out) return fail(c, DG_ERR_INVALID_ARG, "debug_entropy");
  DG_CUDA(c, cudaMemcpyAsync(out, c->dbg_entropy, static_cast<size_t>(c->B) * c->cfg.canvas * 4,
                             cudaMemcpyDeviceToDevice, c->stream));
  return DG_OK;
}

dg_status dg_debug_wait_timeout(dg_ctx* c, uint64_t limit_ns) {
  if (!c || limit_ns == 0 || limit_ns > 10000000000ull) return fail(c, DG_ERR_INVALID_ARG, "wait_timeout");
  wait_timeout_kernel<<<1, 32, 0, c->stream>>>(DevErr{c->err_word, limit_ns});
  DG_LAUNCHED(c);
  return DG_OK;
}

dg_status dg_debug_gemm(dg_ctx* c, const void* w, int32_t M, int32_t K, const void* x, int32_t T, int32_t splits,
                        float* out) {
  if (!c || !w || !x || !out || M <= 0 || T <= 0 || K <= 0 || K % 64 || splits < 1 || splits > K / 64 ||
      !aligned16(w) || !aligned16(x))
    return fail(c, DG_ERR_INVALID_ARG, "debug_gemm");
  GemmParams p;
  memset(&p, 0, sizeof(p));
  if (!make_map(&p.a_map[0], w, M, K, 128) || !make_map(&p.b_map, x, T, K, 64))
    return fail(c, DG_ERR_CUDA, "debug_gemm: tensor map");
  p.b_box_rows = 64;
  p.M = M;
  p.T = T;
  p.k_steps = K / 64;
  p.bn = std::min(DENSE_BN, (T + 15) / 16 * 16);
  p.n_tiles_n = (T + p.bn - 1) / p.bn;
  p.splits = splits;
  p.tiles_static = ((M + GEMM_BM - 1) / GEMM_BM) * p.n_tiles_n * splits;
  if (M % 4) return fail(c, DG_ERR_INVALID_ARG, "debug_gemm: M must be a multiple of 4");
  p.out_f32 = out;
  p.use_tma_store = make_map_partials(&p.out_map, out, splits, T, M) ? 1 : 0;
  p.work = c->dense_work;
  p.err = dev_err(c);
  gemm_kernel<GEMM_DENSE><<<std::min(c->sms, p.tiles_static), GEMM_THREADS, gemm_smem_bytes<GEMM_DENSE>(),
                            c->stream>>>(p);
  DG_LAUNCHED(c);
  return DG_OK;
}

constexpr bool timeline_ids_match() {
  using namespace dg;
  const int ours[17] = {TLK_GEMM + GEMM_DENSE, TLK_GEMM + GEMM_MOE, TLK_GEMM + GEMM_LMHEAD, TLK_ATTENTION, TLK_ATTN_MERGE,
                        TLK_ROUTE_DISPATCH, TLK_COMBINE_NORM, TLK_EMBED_NORM, TLK_RESIDUAL_NORM, TLK_REDUCE_SPLITS,
                        TLK_SWIGLU_SPLITS, TLK_ROPE_QKV, TLK_LMHEAD_MERGE_SAMPLE, TLK_ENTROPY_SAMPLE, TLK_ROUTER_TOPK,
                        TLK_SAMPLE_ONLY, TLK_OTHER};
  const int abi[17] = {DG_K_GEMM_DENSE, DG_K_GEMM_MOE, DG_K_GEMM_LMHEAD, DG_K_ATTENTION, DG_K_ATTN_MERGE, DG_K_ROUTE_DISPATCH,
                       DG_K_COMBINE_NORM, DG_K_EMBED_NORM, DG_K_RESIDUAL_NORM, DG_K_REDUCE_SPLITS, DG_K_SWIGLU_SPLITS,
                       DG_K_ROPE_QKV, DG_K_LMHEAD_MERGE_SAMPLE, DG_K_ENTROPY_SAMPLE, DG_K_ROUTER_TOPK,
                       DG_K_SAMPLE_ONLY, DG_K_OTHER};
  for (int i = 0; i < 17; ++i)
    if (ours[i] != abi[i]) return false;
  return true;
}
static_assert(timeline_ids_match(), "timeline kernel ids match the ABI");

dg_status dg_debug_timeline_reset(dg_ctx* c) {
  if (!c) return DG_ERR_INVALID_ARG;
#ifdef DG_TIMELINE
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  const unsigned int zero = 0;
  DG_CUDA(c, cudaMemcpyToSymbol(dg::g_timeline_n, &zero, sizeof(zero)));
  return DG_OK;
#else
  return fail(c, DG_ERR_UNSUPPORTED, "this library was built without the timeline (see libdg_timeline.so)");
#endif
}

dg_status dg_debug_timeline(dg_ctx* c, dg_timeline_record* host, int32_t capacity, int64_t* n_records) {
  if (!c || !n_records || capacity < 0 || (capacity > 0 && !host)) return DG_ERR_INVALID_ARG;
#ifdef DG_TIMELINE
  static_assert(sizeof(dg_timeline_record) == sizeof(dg::TimelineRecord), "record layout");
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  unsigned int n = 0;
  DG_CUDA(c, cudaMemcpyFromSymbol(&n, dg::g_timeline_n, sizeof(n)));
  *n_records = n;
  const size_t m = std::min<size_t>({static_cast<size_t>(n), static_cast<size_t>(capacity),
                                     static_cast<size_t>(dg::TIMELINE_CAP)});
  if (m > 0) DG_CUDA(c, cudaMemcpyFromSymbol(host, dg::g_timeline, m * sizeof(dg_timeline_record)));
  return DG_OK;
#else
  (void)host;
  *n_records = 0;
  return fail(c, DG_ERR_UNSUPPORTED, "this library was built without the timeline (see libdg_timeline.so)");
#endif
}

dg_status dg_debug_profile(dg_ctx* c, int32_t mask) {
  if (!c) return DG_ERR_INVALID_ARG;
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  for (auto& v : c->prof_pairs) v.clear();
  c->ev_used = 0;
  c->prof_mask = mask;
  return DG_OK;
}

dg_status dg_debug_profile_read(dg_ctx* c, int32_t cls, double* total_ms, int64_t* launches) {
  if (!c || cls < 0 || cls >= DG_PROF_CLASSES || !total_ms || !launches)
    return fail(c, DG_ERR_INVALID_ARG, "profile_read");
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  double t = 0.0;
  for (auto& pr : c->prof_pairs[cls]) {
    float ms = 0.f;
    DG_CUDA(c, cudaEventElapsedTime(&ms, pr.first, pr.second));
    t += ms;
  }
  *total_ms = t;
  *launches = static_cast<int64_t>(c->prof_pairs[cls].size());
  return DG_OK;
}

int64_t dg_debug_launch_count(const dg_ctx* c) { return c ? c->launches : -1; }

}  // extern "C"

// =============================================================================
// LM-head reduction that allocates nothing (dg_lmhead_argmax_static).
//
// Some callers cannot allocate device memory at the time they need this: code
// that runs while another framework records a CUDA graph (allocation is not
// allowed inside the capture), processes whose caching allocator has already
// reserved the whole device, or embedded deployments that fix every byte of
// device memory at start-up.  For them the per-(vocabulary tile, row)
// partials of the LM-head reduction live in a fixed array in the library's
// own device image instead of a context workspace.
// =============================================================================
namespace {

constexpr size_t kLmStaticPartials = 524288;  // float4 entries = 8 MiB: n_rows * vocab / 128 <= this

// Shared by every call on a device (the library image holds it until exit).
static __device__ __align__(256) float4 g_lm_static_partials[kLmStaticPartials];
static __device__ __align__(256) int g_lm_static_err[4];

constexpr int kMaxDevices = 64;
struct StaticSetup {
  bool done = false;
  float4* partials = nullptr;  // device address of g_lm_static_partials on this device
  int* err = nullptr;          // device address of g_lm_static_err on this device
  int sms = 0;
};
StaticSetup g_static_setup[kMaxDevices];
std::mutex g_static_setup_mutex;  // the first calls on a device may come from several threads

// merge of the partials into argmax / lse / conf (rows flagged by a timed-out
// wait get argmax -1 and NaN statistics)
__global__ void lmhead_static_merge_kernel(const float4* __restrict__ part, int n_vtiles, int T,
                                           const int* __restrict__ err, int32_t* __restrict__ argmax,
                                           float* __restrict__ lse, float* __restrict__ conf) {
  DG_TIMELINE_SCOPE(dg::TLK_OTHER);
  const int t = blockIdx.x;
  const Top2 acc = merge_token_partials(part, nullptr, n_vtiles, T, t);
  if (threadIdx.x == 0) {
    const bool bad = err[0] != 0;
    if (argmax) argmax[t] = bad ? -1 : acc.idx;
    if (lse) lse[t] = bad ? NAN : (acc.m1 + log2f(acc.s)) * 0.69314718055994531f;
    if (conf) conf[t] = bad ? NAN : 1.f / acc.s;
  }
}

}  // namespace

extern "C" dg_status dg_lmhead_argmax_static(const void* z, int32_t n_rows, int32_t d_model, const void* embed,
                                             int32_t vocab, float temperature, int32_t* argmax_out,
                                             float* lse_out, float* conf_out, void* cuda_stream) {
  if (!z || !embed || n_rows <= 0 || d_model <= 0 || d_model % 64 || vocab <= 0 || vocab % GEMM_BN ||
      !(temperature > 0.f) || !aligned16(z) || !aligned16(embed) || (!argmax_out && !lse_out && !conf_out))
    return DG_ERR_INVALID_ARG;
  const int n_vtiles = vocab / GEMM_BN;
  if (static_cast<size_t>(n_vtiles) * static_cast<size_t>(n_rows) > kLmStaticPartials)
    return DG_ERR_CAPACITY;  // n_rows * vocab / 128 beyond the fixed scratch
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DG_ERR_CUDA;
  StaticSetup su;
  {
    // once per device, with that device current (the caller's current device)
    std::lock_guard<std::mutex> lock(g_static_setup_mutex);
    StaticSetup& g = g_static_setup[dev];
    if (!g.done) {
      StaticSetup n;
      if (cudaGetSymbolAddress(reinterpret_cast<void**>(&n.partials), g_lm_static_partials) != cudaSuccess ||
          cudaGetSymbolAddress(reinterpret_cast<void**>(&n.err), g_lm_static_err) != cudaSuccess ||
          cudaDeviceGetAttribute(&n.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
          cudaFuncSetAttribute(gemm_kernel<GEMM_LMHEAD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               gemm_smem_bytes<GEMM_LMHEAD>()) != cudaSuccess)
        return DG_ERR_CUDA;
      n.done = true;
      g = n;
    }
    su = g;
  }
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  GemmParams p;
  memset(&p, 0, sizeof(p));
  if (!make_map(&p.a_map[0], z, n_rows, d_model, 128) || !make_map(&p.b_map, embed, vocab, d_model, 128))
    return DG_ERR_CUDA;
  p.b_box_rows = 128;
  p.M = n_rows;
  p.k_steps = d_model / 64;
  p.n_mtiles = (n_rows + GEMM_BM - 1) / GEMM_BM;
  p.tiles_static = n_vtiles * lmhead_mpairs(p.n_mtiles);
  p.lm_part = su.partials;
  p.logit_scale_log2 = static_cast<float>(1.4426950408889634 / static_cast<double>(temperature));
  p.err = DevErr{su.err, 1000000000ull};
  if (cudaMemsetAsync(su.err, 0, sizeof(int), st) != cudaSuccess) return DG_ERR_CUDA;
  // each launch's own status (cudaLaunchKernelEx), so an error the caller
  // left pending from its own earlier work is neither reported nor cleared here
  cudaLaunchConfig_t lc{};
  lc.gridDim = dim3(std::min(su.sms, p.tiles_static));
  lc.blockDim = dim3(GEMM_THREADS);
  lc.dynamicSmemBytes = gemm_smem_bytes<GEMM_LMHEAD>();
  lc.stream = st;
  if (cudaLaunchKernelEx(&lc, gemm_kernel<GEMM_LMHEAD>, p) != cudaSuccess) return DG_ERR_CUDA;
  lc.gridDim = dim3(n_rows);
  lc.blockDim = dim3(256);
  lc.dynamicSmemBytes = 0;
  const float4* parts = su.partials;
  const int* errp = su.err;
  if (cudaLaunchKernelEx(&lc, lmhead_static_merge_kernel, parts, n_vtiles, static_cast<int>(n_rows), errp,
                         argmax_out, lse_out, conf_out) != cudaSuccess)
    return DG_ERR_CUDA;
  return DG_OK;
}
