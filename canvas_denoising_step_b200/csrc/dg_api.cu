// C ABI of libdg: argument checks, device memory, weight initialisation and
// the orchestration of one canvas denoising pass on a single stream.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <string>
#include <vector>

#include "dg.h"
#include "dg_kernels.h"

using namespace dg;

namespace {

#ifndef DG_GROUPED_TILE
#define DG_GROUPED_TILE 256
#endif
constexpr int kGroupedTile = DG_GROUPED_TILE;   // rows of an expert chunk (B rows per grouped tile)
#ifndef DG_GROUPED_BOX
#define DG_GROUPED_BOX 64
#endif

constexpr int kGroupedBox = DG_GROUPED_BOX;   // B rows per TMA box of a grouped tile
#ifndef DG_DOWN_PAIR
#define DG_DOWN_PAIR 1
#endif
constexpr bool kDownPair = DG_DOWN_PAIR != 0;
constexpr int kMaxAttnChunks = 16;
constexpr int kMaxSplits = 16;
// entropy-bounded denoising settings ("DiffusionGemma: The Diffusion Era Begins with
// 4x Faster Text Generation", Recommended Inference Settings)
constexpr double kEbBound = 0.1;          // entropy bound per pass (nats)
constexpr double kEbStopEntropy = 0.005;  // mean canvas entropy that allows a stop
constexpr double kEbTempStart = 0.8, kEbTempEnd = 0.4;

std::string g_create_error;

struct Layer {
  bf16 *wqkv = nullptr, *wo = nullptr, *wr = nullptr, *wgu = nullptr, *wd = nullptr;
  // FP8 expert weights (expert_dtype = DG_DTYPE_FP8_E4M3): codes and row scales
  uint8_t *wgu8 = nullptr, *wd8 = nullptr;
  float *sgu = nullptr, *sd8 = nullptr;
  CUtensorMap m_gu8, m_d8;
  float *ln_in = nullptr, *ln_post = nullptr, *ln_ff = nullptr;
  CUtensorMap m_qkv, m_o, m_r, m_gu, m_d;
  CUtensorMap m_kp, m_vp;   // prompt K/V of this layer, 64-row boxes
  const bf16* kp = nullptr;
  const bf16* vp = nullptr;
  int kv_batch = 0, kv_P = 0;
  int kv_stride = 0;   // rows per (sequence, kv head) behind m_kp / m_vp
  // the library's own KV cache (max_context > 0): [max_batch][Hkv][max_context][dh]
  bf16 *own_k = nullptr, *own_v = nullptr;
};

}  // namespace

struct dg_ctx {
  dg_config cfg;
  cudaStream_t stream = nullptr;
  int device = 0, num_sms = 148;
  std::string err;
  size_t bytes = 0;
  std::vector<void*> allocs;
  bool weights_ready = false;

  int Tmax = 0, NQKV = 0, G = 0;
  int dense_box = 256;   // B rows per dense-GEMM tile: one TMA box covers all canvas rows
  bf16* embed = nullptr;
  float* ln_final = nullptr;
  std::vector<Layer> layers;
  CUtensorMap m_embed;

  // workspace
  float* h = nullptr;
  bf16* x = nullptr;
  float* part = nullptr;
  size_t part_elems = 0;
  bf16 *q = nullptr, *kc = nullptr, *vc = nullptr;
  float *attn_po = nullptr, *attn_ml = nullptr;
  bf16* attn_o = nullptr;
  bf16* xperm = nullptr;
  float* router_logits = nullptr;
  int32_t* idx = nullptr;
  float* w = nullptr;
  uint32_t* bitmap = nullptr;
  int* router_counter = nullptr;
  int chunk_rows = 0;                // rows of an expert chunk (B rows per grouped tile)
  int* chunk_ready = nullptr;        // per-chunk gate/up -> down hand-over counters
  int n_chunk_ready = 0;
  int32_t* chunk_order = nullptr;    // [n_chunk_ready] the expert chunks longest first
  int* tile_counters = nullptr;      // [2] the gate/up and down GEMMs' dynamic tile counters
  int32_t *offsets_r = nullptr, *offsets_g = nullptr, *chunk_prefix = nullptr;
  int32_t *perm = nullptr, *inv = nullptr;
  bf16* H = nullptr;
  float* Y = nullptr;
  float *head_m = nullptr, *head_s = nullptr;
  int* head_a = nullptr;
  float* conf = nullptr;
  float* head_max = nullptr;       // largest logit per row (mask id excluded)
  // entropy-bounded passes
  float* head_q = nullptr;         // [V/256][T] sum z e^z per vocab block
  float* eb_H = nullptr;           // [T] entropy per row
  float* eb_sum = nullptr;         // [T] sum e^((l - max) / temp)
  float* eb_u = nullptr;           // [T] the pass's uniforms
  int32_t* eb_prev = nullptr;      // [T] previous pass's argmax
  int32_t* eb_drawn = nullptr;     // [T] drawn token of each committed slot
  int* eb_state = nullptr;         // [Bmax] bit 0: eb_prev valid, bit 1: done
  uint8_t* eb_stopped = nullptr;   // [Bmax]
  float* eb_inv_temp = nullptr;    // 1 / temperature of the pass
  int* eb_last = nullptr;          // the pass is the last allowed one
  int32_t* tok = nullptr;
  int32_t* canvas_dev = nullptr;
  uint8_t* committed_dev = nullptr;
  int* err_dev = nullptr;
  int* expert_active = nullptr;   // [n_layers] cumulative count of experts given rows
  float *rope_cos = nullptr, *rope_sin = nullptr;
  int rope_P = -1;
  float* router_bias = nullptr;
  bool has_bias = false;
  CUtensorMap m_x_b, m_x_a, m_attn_o_b, m_xperm_b, m_H_b, m_x2_b;
  // half-height B boxes (dense_box / 2 rows) of the two-SM dense projections
  CUtensorMap m_x_bh, m_attn_o_bh;
  // Two-SM (cta_group::2) q/k/v, o and bf16 expert GEMMs, when the environment
  // sets DG_CTA_PAIR=1: co-resident two-CTA clusters, 0 when off.  Measured
  // slower than the one-SM engine on every workload here, so off by default.
  int pair_clusters = 0;
  // the router with its logits GEMM in one cluster kernel, when the environment sets
  // DG_FUSED_ROUTER=1: parity-green, but the pass measured slower than with the logits
  // GEMM and the router kernel apart (6.72 vs 6.56 ms on the stack), so off by default
  bool fused_router = false;
  // The attention's key ranges merged inside a thread-block cluster (no partials
  // through global memory, no merge kernel), when the environment sets
  // DG_ATTN_CLUSTER_MERGE=1.  Both routes give the same bits; on the stack the
  // cluster route measured slower (6.66 against 6.57 ms per pass: its merge phase
  // adds ~7 µs to each attention launch, while the merge kernel it replaces costs
  // less than that inside the graph), so the merge kernel is the default.
  bool attn_cluster_merge = false;
  // Encoded context in the library's own KV cache (dg_encode / dg_generate):
  // positions held, and the batch they belong to (0: none yet).
  int ctx_len = 0, ctx_batch = 0;
  int32_t* gen_canvas = nullptr;   // [max_batch][canvas_len] working canvas of dg_generate
  CUtensorMap m_Y_out;   // fp32 expert outputs [1][rows][d], tensor-store map
  CUtensorMap m_H_out;   // bf16 gate/up outputs [rows][F], tensor-store map
  CUtensorMap m_q, m_kc, m_vc;   // attention operands
  CUtensorMap m_attn_po;         // attention partial outputs (tensor stores)

  int last_T = 0, last_B = 0, launches = 0;
  int* steps_dev = nullptr;          // steps_left of the pass being run
  struct StepGraph { cudaGraphExec_t exec = nullptr; int launches = 0; };
  std::map<int, StepGraph> graphs;   // captured passes, by 2 * batch size + (entropy-bounded)
  std::map<int, bool> warm;
  struct ProfRec { int kind; cudaEvent_t a, b; };
  bool prof_on = false;
  std::vector<ProfRec> prof;
  std::vector<cudaEvent_t> ev_pool;
};

namespace {

int fail(dg_ctx* c, int code, const std::string& msg) {
  if (c) c->err = msg;
  else g_create_error = msg;
  return code;
}

#define DG_CUDA(ctx, call)                                                             \
  do {                                                                                 \
    cudaError_t e_ = (call);                                                           \
    if (e_ != cudaSuccess)                                                             \
      return fail(ctx, DG_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)

#define DG_LAUNCH(ctx, kind, call)          \
  do {                                      \
    ++(ctx)->launches;                      \
    const int pi_ = prof_begin(ctx, kind);  \
    DG_CUDA(ctx, call);                     \
    prof_end(ctx, pi_);                     \
  } while (0)

enum KernelKind {
  K_EMBED, K_ROPE_TABLE, K_GEMM_QKV, K_ROPE, K_ATTN, K_ATTN_MERGE, K_GEMM_O, K_POST_ATTN,
  K_GEMM_ROUTER, K_ROUTER, K_GATHER, K_GEMM_GATEUP, K_GEMM_DOWN, K_COMBINE,
  K_GEMM_HEAD, K_HEAD_MERGE, K_COMMIT, K_KV_APPEND, K_NUM_KINDS
};
const char* const kKindNames[K_NUM_KINDS] = {
  "embed_norm", "rope_table", "gemm_qkv", "qkv_rope", "attention", "attn_merge", "gemm_o",
  "post_attn", "gemm_router", "router", "moe_gather", "gemm_gateup",
  "gemm_down", "moe_combine", "gemm_head", "head_merge", "commit", "kv_append"};

// Per-launch CUDA events while profiling is on (events come from a growing pool).
int prof_begin(dg_ctx* c, int kind) {
  if (!c->prof_on) return -1;
  const size_t need = 2 * (c->prof.size() + 1);
  while (c->ev_pool.size() < need) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return -1;
    c->ev_pool.push_back(e);
  }
  const int i = (int)c->prof.size();
  c->prof.push_back({kind, c->ev_pool[2 * i], c->ev_pool[2 * i + 1]});
  cudaEventRecord(c->prof[i].a, c->stream);
  return i;
}

void prof_end(dg_ctx* c, int i) {
  if (i >= 0) cudaEventRecord(c->prof[i].b, c->stream);
}

bool ctx_alloc(dg_ctx* c, void** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) bytes = 16;
  bytes = (bytes + 255) & ~size_t(255);
  if (c->cfg.alloc_limit_bytes && c->bytes + bytes > c->cfg.alloc_limit_bytes) return false;
  if (cudaMalloc(p, bytes) != cudaSuccess) {
    *p = nullptr;
    cudaGetLastError();
    return false;
  }
  c->allocs.push_back(*p);
  c->bytes += bytes;
  return true;
}

template <class T>
bool alloc_n(dg_ctx* c, T** p, size_t n) {
  return ctx_alloc(c, reinterpret_cast<void**>(p), n * sizeof(T));
}

void free_all(dg_ctx* c) {
  for (void* p : c->allocs) cudaFree(p);
  c->allocs.clear();
}

bool is_global(const dg_config& c, int l) { return (l + 1) % c.global_every == 0; }

int n_rot_pairs(const dg_config& c, int l) {
  if (!c.rope_enabled) return 0;
  const int half = c.head_dim / 2;
  if (is_global(c, l)) return (int)std::ceil((double)c.prope_fraction * half);
  return half;
}

std::string check_config(const dg_config& c) {
  if (c.n_layers < 1) return "n_layers must be >= 1";
  if (c.d_model < 128 || c.d_model % 64 || c.d_model > 4096) return "d_model must be a multiple of 64 in [128, 4096]";
  if (c.d_ff < 64 || c.d_ff % 64) return "d_ff must be a positive multiple of 64";
  if (c.head_dim != 64 && c.head_dim != 128 && c.head_dim != 256) return "head_dim must be 64, 128 or 256";
  if (c.n_kv_heads < 1 || c.n_q_heads < 1 || c.n_q_heads % c.n_kv_heads) return "n_q_heads must be a positive multiple of n_kv_heads";
  if (c.n_experts < 4 || c.n_experts > 256 || c.n_experts % 4) return "n_experts must be a multiple of 4 in [4, 256]";
  if (c.top_k < 1 || c.top_k > c.n_experts || c.top_k > 32) return "top_k must be in [1, min(n_experts, 32)]";
  if ((c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim > 16384) return "(n_q_heads + 2 n_kv_heads) * head_dim must be <= 16384";
  if (c.n_shared != 0 && c.n_shared != 1) return "n_shared must be 0 or 1";
  if (c.vocab < 2) return "vocab must be >= 2";
  if (c.canvas_len < 1 || c.canvas_len > 256) return "canvas_len must be in [1, 256]";
  if (c.max_batch < 1 || (long long)c.max_batch * c.canvas_len > 4096) return "max_batch * canvas_len must be in [1, 4096]";
  if (c.max_prompt < 1) return "max_prompt must be >= 1";
  if (c.max_context < 0) return "max_context must be >= 0";
  if (c.mask_id < 0 || c.mask_id >= c.vocab) return "mask_id must be in [0, vocab)";
  if (c.window < 1 || c.global_every < 1) return "window and global_every must be >= 1";
  if (!(c.rms_eps >= 0.f) || !(c.rope_theta > 0.f)) return "rms_eps must be >= 0 and rope_theta > 0";
  if (!(c.prope_fraction >= 0.f && c.prope_fraction <= 1.f)) return "prope_fraction must be in [0, 1]";
  if (!(c.weight_std > 0.0)) return "weight_std must be > 0";
  if (c.expert_dtype != DG_DTYPE_BF16 && c.expert_dtype != DG_DTYPE_FP8_E4M3)
    return "expert_dtype must be DG_DTYPE_BF16 or DG_DTYPE_FP8_E4M3";
  // the router groups all rows of a pass in one CTA's shared memory
  if (router_smem_bytes(c.max_batch * c.canvas_len, c.n_experts) >
      (size_t)router_max_smem_bytes())
    return "max_batch * canvas_len rows with n_experts experts exceed the router's shared "
           "memory (2 * n_experts * ceil(rows / 32) + 2 * n_experts + 1 words <= 200 KB)";
  return "";
}

int choose_splits(int base_tiles, int n_kb, int num_sms) {
  int best = 1;
  double best_cost = 1e30;
  for (int ks = 1; ks <= kMaxSplits && ks <= n_kb; ++ks) {
    const int tiles = base_tiles * ks;
    const int waves = (tiles + num_sms - 1) / num_sms;
    const double cost = (double)waves / ks * (1.0 + 0.02 * ks);  // small penalty for partial traffic
    if (cost < best_cost - 1e-9) { best_cost = cost; best = ks; }
  }
  return best;
}

// Dense swap-AB projection: part[s][n][m] = X[n] . W[m] over split s.  With
// mB_half (the same activation in half-height boxes) and an even number of
// weight slabs, tile pairs run on two-SM clusters (gemm_pair.cu).
int run_dense(dg_ctx* c, int kind, const CUtensorMap& mA, const CUtensorMap& mB,
              const CUtensorMap* mB_half, int M, int N, int K, int* splits_out) {
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.mode = GEMM_DENSE;
  a.M = M; a.N = N; a.K = K; a.n_kb = K / 64;
  a.n_tile = c->dense_box;      // one B box per stage covers the activation rows
  a.b_box_rows = c->dense_box;
  // one 128-row weight slab per tile: pairing two slabs over one activation tile
  // (dense_pair) measured slower here (6.73 -> 7.30 ms per stack pass)
  a.m_slabs = (M + 127) / 128;
  const int n_chunks = (N + a.n_tile - 1) / a.n_tile;
  a.k_splits = choose_splits(a.m_slabs * n_chunks, a.n_kb, c->num_sms);
  if ((size_t)a.k_splits * N * M > c->part_elems) a.k_splits = 1;
  a.out_f32 = c->part;
  a.err = c->err_dev;
  gemm_plan_smem(a);
  // the split-K partials [k_splits][N][M], written by tensor stores
  CUtensorMap mC;
  if (!make_tmap_out_f32(&mC, c->part, (uint64_t)M, (uint64_t)N, (uint64_t)a.k_splits))
    return fail(c, DG_ERR_CUDA, "tensor map for a projection output failed");
  const int tiles = a.m_slabs * n_chunks * a.k_splits;
  if (mB_half && c->pair_clusters > 0 && a.m_slabs % 2 == 0) {
    a.b_box_rows = c->dense_box / 2;
    gemm_pair_plan_smem(a);
    DG_LAUNCH(c, kind, gemm_pair_launch(mA, *mB_half, mC, a, std::min(tiles / 2, c->pair_clusters),
                                        c->stream));
  } else {
    DG_LAUNCH(c, kind, gemm_tc_launch(mA, mB, mC, a, std::min(tiles, c->num_sms), c->stream));
  }
  *splits_out = a.k_splits;
  return DG_OK;
}

int run_grouped(dg_ctx* c, const Layer& L, int mode, const CUtensorMap& mB, int K, int M) {
  const dg_config& cf = c->cfg;
  const bool fp8 = L.wgu8 != nullptr;
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.mode = mode;
  a.K = K; a.n_kb = K / 64;
  a.M = M;
  a.n_tile = c->chunk_rows;
  a.b_box_rows = kGroupedBox;
  // down: 256 weight rows per tile (its H chunk is read once per two slabs); the
  // FP8-weight GEMMs keep one slab a tile to leave room for their deeper rings
  const bool cta_pair = !fp8 && c->pair_clusters > 0;
  a.pair = !fp8 && !cta_pair && mode == GEMM_DOWN && kDownPair ? 1 : 0;
  a.m_slabs = a.pair ? (M + 255) / 256 : (M + 127) / 128;
  // two-SM tiles pair slabs 2p and 2p + 1: an odd slab count gets one empty
  // slab (its weight rows read as zeros, its outputs are not stored)
  if (cta_pair) a.m_slabs += a.m_slabs & 1;
  a.chunk_order = c->chunk_order;
  a.max_chunks = c->n_chunk_ready;
  a.tile_counter = c->tile_counters + (mode == GEMM_DOWN ? 1 : 0);
  a.n_groups = cf.n_experts + 1;
  a.offsets = c->offsets_g;
  a.chunk_prefix = c->chunk_prefix;
  a.F = cf.d_ff;
  a.out_f32 = c->Y;
  a.out_bf16 = c->H;
  a.err = c->err_dev;
  // gate/up hands each chunk's H rows to down as soon as its slabs are written
  a.chunk_ready = c->chunk_ready;
  // epilogue warps x gate/up slabs of a chunk (as gate/up counts them)
  const int gu_slabs = (2 * cf.d_ff + 127) / 128;
  a.ready_target = 4 * (cta_pair ? gu_slabs + (gu_slabs & 1) : gu_slabs);
  const int kind = mode == GEMM_GATEUP ? K_GEMM_GATEUP : K_GEMM_DOWN;
  const CUtensorMap& mC = mode == GEMM_GATEUP ? c->m_H_out : c->m_Y_out;
  if (fp8) {
    a.w_scale = mode == GEMM_GATEUP ? L.sgu : L.sd8;
    gemm_fp8_plan_smem(a);
    DG_LAUNCH(c, kind, gemm_fp8_launch(mode == GEMM_GATEUP ? L.m_gu8 : L.m_d8, mB, mC, a,
                                       c->num_sms, c->stream));
  } else if (cta_pair) {
    gemm_pair_plan_smem(a);
    DG_LAUNCH(c, kind, gemm_pair_launch(mode == GEMM_GATEUP ? L.m_gu : L.m_d, mB, mC, a,
                                        c->pair_clusters, c->stream));
  } else {
    gemm_plan_smem(a);
    DG_LAUNCH(c, kind, gemm_tc_launch(mode == GEMM_GATEUP ? L.m_gu : L.m_d, mB, mC, a, c->num_sms,
                                      c->stream));
  }
  return DG_OK;
}

// FP8 codes and row scales of one layer's expert weights, from its bf16 weights.
int quantize_layer(dg_ctx* c, Layer& L) {
  if (!L.wgu8) return DG_OK;
  const dg_config& cf = c->cfg;
  const long long G = c->G, F = cf.d_ff, d = cf.d_model;
  DG_CUDA(c, launch_quantize_rows(L.wgu, L.wgu8, L.sgu, G * 2 * F, (int)d, c->stream));
  DG_CUDA(c, launch_quantize_rows(L.wd, L.wd8, L.sd8, G * d, (int)F, c->stream));
  return DG_OK;
}

// One block on c->h / c->x (x = input-normed h) for B sequences of Tc rows.  On
// return h is the block output and x = bf16(rmsnorm(h) * w_next) (or bf16(h)
// when w_next is NULL).  The decoder (causal false) attends jointly over the
// visible prompt keys and all Tc canvas keys; the encoder (causal true) attends
// causally over the cached positions and the Tc new tokens, then appends the
// new tokens' keys and values to the layer's own cache at positions P ...
int run_layer(dg_ctx* c, int l, int B, const float* w_next, int Tc, bool causal) {
  const dg_config& cf = c->cfg;
  Layer& L = c->layers[l];
  const int T = B * Tc, d = cf.d_model, dh = cf.head_dim;
  const int Hq = cf.n_q_heads, Hkv = cf.n_kv_heads, E = cf.n_experts, k = cf.top_k;
  const int P = L.kv_P;
  int splits = 1, rc;

  // q/k/v projections, RoPE / p-RoPE on the canvas rows
  if ((rc = run_dense(c, K_GEMM_QKV, L.m_qkv, c->m_x_b, &c->m_x_bh, c->NQKV, T, d, &splits)) != DG_OK) return rc;
  DG_LAUNCH(c, K_ROPE, launch_qkv_rope(c->part, splits, T, Tc, Hq, Hkv, dh, n_rot_pairs(cf, l), c->rope_cos,
                               c->rope_sin, c->q, c->kc, c->vc, c->stream));

  // one softmax over the visible prompt keys and all canvas keys, split-KV
  AttnTcArgs ta;
  memset(&ta, 0, sizeof(ta));
  ta.B = B; ta.Hq = Hq; ta.Hkv = Hkv; ta.Tc = Tc; ta.P = P; ta.dh = dh;
  ta.kv_stride = L.kv_stride;
  if (!causal) {
    ta.n_vis = is_global(cf, l) ? P : std::min(cf.window, P);
  } else {
    // new token 0 (position P) sees the last window - 1 cached positions
    ta.causal = 1;
    ta.window = is_global(cf, l) ? 0 : cf.window;
    ta.n_vis = is_global(cf, l) ? P : std::min(cf.window - 1, P);
  }
  {
    // key-block ranges per (canvas, kv head, query tile): about one CTA per SM
    const int nb = attn_tc_blocks(ta.n_vis, Tc);
    const int base = attn_tc_qtiles(Hq, Hkv, Tc) * B * Hkv;
    ta.n_chunks = std::max(1, std::min({kMaxAttnChunks, nb, c->num_sms / base}));
  }
  ta.part_o = c->attn_po; ta.part_ml = c->attn_ml;
  ta.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)dh));
  ta.err = c->err_dev;
  ta.out = c->attn_o;
  ta.fused = (c->attn_cluster_merge && attn_tc_fused_ok(dh, ta.n_chunks)) ? 1 : 0;
  AttnTcMaps tm;
  tm.q = c->m_q; tm.kc = c->m_kc; tm.vc = c->m_vc; tm.kp = L.m_kp; tm.vp = L.m_vp;
  tm.po = c->m_attn_po;
  DG_LAUNCH(c, K_ATTN, launch_attention_tc(tm, ta, c->stream));
  if (!ta.fused) {
    AttnMergeArgs at;
    at.B = B; at.Hq = Hq; at.Tc = Tc; at.dh = dh;
    at.n_chunks = ta.n_chunks;
    at.part_o = c->attn_po; at.part_ml = c->attn_ml;
    DG_LAUNCH(c, K_ATTN_MERGE, launch_attn_merge(at, c->attn_o, c->stream));
  }
  if (causal)
    DG_LAUNCH(c, K_KV_APPEND, launch_kv_append(c->kc, c->vc, L.own_k, L.own_v, B, Hkv, Tc, dh,
                                               cf.max_context, P, c->stream));

  // output projection, post-attention norm + residual, pre-FFN norm
  if ((rc = run_dense(c, K_GEMM_O, L.m_o, c->m_attn_o_b, &c->m_attn_o_bh, d, T, Hq * dh, &splits)) != DG_OK) return rc;
  DG_LAUNCH(c, K_POST_ATTN, launch_post_attn(c->part, splits, T, d, L.ln_post, L.ln_ff, cf.rms_eps, c->h,
                                c->xperm, c->stream));

  // router: logits, top-k and grouping in one cluster kernel (E <= 128), or the
  // logits GEMM then the router kernel
  const bool fused_router = c->fused_router && E <= 128;
  if (!fused_router &&
      (rc = run_dense(c, K_GEMM_ROUTER, L.m_r, c->m_x2_b, nullptr, E, T, d, &splits)) != DG_OK)
    return rc;
  {
    RouterArgs ra;
    memset(&ra, 0, sizeof(ra));
    ra.logits_in = c->part; ra.splits = splits;
    ra.bias = c->has_bias ? c->router_bias : nullptr;
    ra.T = T; ra.E = E; ra.k = k; ra.n_shared = cf.n_shared; ra.n_tile = c->chunk_rows;
    ra.logits_out = c->router_logits; ra.idx = c->idx; ra.w = c->w;
    ra.bitmap = c->bitmap; ra.counter = c->router_counter;
    ra.offsets_r = c->offsets_r; ra.offsets_g = c->offsets_g; ra.chunk_prefix = c->chunk_prefix;
    ra.chunk_ready = c->chunk_ready; ra.n_chunk_ready = c->n_chunk_ready;
    ra.chunk_order = c->chunk_order; ra.tile_counters = c->tile_counters; ra.n_tile_counters = 2;
    ra.perm = c->perm; ra.inv = c->inv; ra.active_out = c->expert_active + l; ra.err = c->err_dev;
    if (fused_router) {
      RouterFusedArgs rf;
      memset(&rf, 0, sizeof(rf));
      rf.r = ra;
      rf.n_kb = d / 64;
      rf.n_tile = c->dense_box;
      DG_LAUNCH(c, K_ROUTER, launch_router_fused(L.m_r, c->m_x2_b, rf, c->stream));
    } else {
      DG_LAUNCH(c, K_ROUTER, launch_router(ra, c->stream));
    }
  }
  DG_LAUNCH(c, K_GATHER, launch_moe_gather(c->xperm, c->perm, T, k, d, c->stream));

  // experts (group 0 = shared expert on all rows), SiLU-gated, then down + combine
  if ((rc = run_grouped(c, L, GEMM_GATEUP, c->m_xperm_b, d, 2 * cf.d_ff)) != DG_OK) return rc;
  if ((rc = run_grouped(c, L, GEMM_DOWN, c->m_H_b, cf.d_ff, d)) != DG_OK) return rc;
  DG_LAUNCH(c, K_COMBINE, launch_moe_combine(c->Y, c->w, c->inv, T, k, cf.n_shared, d, c->h, w_next,
                                  cf.rms_eps, c->x, c->stream));
  return DG_OK;
}

int check_prompt_state(dg_ctx* c, int batch) {
  const dg_config& cf = c->cfg;
  int P = -1;
  for (int l = 0; l < cf.n_layers; ++l) {
    const Layer& L = c->layers[l];
    if (!L.kp) return fail(c, DG_ERR_BAD_STATE, "prompt KV not set for layer " + std::to_string(l));
    if (L.kv_batch != batch)
      return fail(c, DG_ERR_BAD_STATE, "batch differs from the batch of the prompt KV");
    if (P >= 0 && L.kv_P != P)
      return fail(c, DG_ERR_BAD_STATE, "all layers need the same prompt length");
    P = L.kv_P;
  }
  return DG_OK;
}

int ensure_rope(dg_ctx* c, int P) {
  if (c->rope_P != P) {
    // positions P .. P + Tmax - 1: a canvas, or an encoder chunk of up to Tmax rows
    DG_LAUNCH(c, K_ROPE_TABLE, launch_rope_table(c->rope_cos, c->rope_sin, c->Tmax,
                                   c->cfg.head_dim / 2, P, (double)c->cfg.rope_theta, c->stream));
    c->rope_P = P;
  }
  return DG_OK;
}

// The kernels of one pass on c->canvas_dev (batch B).  Fixed-step pass: conf/tok
// into c->conf / c->tok, commit in place with steps_left read from c->steps_dev.
// Entropy-bounded pass (eb): the head at temperature 1 / *c->eb_inv_temp, entropy
// and argmax into c->eb_H / c->tok, then the stop test and the bounded commit
// with the uniforms in c->eb_u.
int record_step(dg_ctx* c, int B, bool eb) {
  const dg_config& cf = c->cfg;
  const int T = B * cf.canvas_len, d = cf.d_model;
  int rc;
  c->launches = 0;
  DG_LAUNCH(c, K_EMBED, launch_embed_norm(c->canvas_dev, c->embed, nullptr, cf.vocab, T, d,
                                 c->layers[0].ln_in, cf.rms_eps, c->h, c->x, c->err_dev,
                                 c->stream));
  for (int l = 0; l < cf.n_layers; ++l) {
    const float* w_next = (l + 1 < cf.n_layers) ? c->layers[l + 1].ln_in : c->ln_final;
    if ((rc = run_layer(c, l, B, w_next, cf.canvas_len, false)) != DG_OK) return rc;
  }
  // tied vocab head with the fused (max, argmax, sum-exp) reduction
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.mode = GEMM_HEAD;
  a.K = d; a.n_kb = d / 64;
  a.T = T; a.vocab = cf.vocab; a.mask_id = cf.mask_id;
  a.n_vblocks = (cf.vocab + 255) / 256;
  a.n_tblocks = (T + 255) / 256;
  a.head_m = c->head_m; a.head_s = c->head_s; a.head_a = c->head_a;
  if (eb) { a.inv_temp = c->eb_inv_temp; a.head_q = c->head_q; }
  a.err = c->err_dev;
  gemm_plan_smem(a);
  const int tiles = a.n_vblocks * a.n_tblocks;
  DG_LAUNCH(c, K_GEMM_HEAD, gemm_tc_launch(c->m_x_a, c->m_embed, c->m_Y_out, a,
                                           std::min(tiles, c->num_sms), c->stream));
  if (!eb) {
    DG_LAUNCH(c, K_HEAD_MERGE, launch_head_merge(c->head_m, c->head_s, c->head_a, a.n_vblocks, T,
                                                 c->conf, c->tok, c->head_max, c->stream));
    DG_LAUNCH(c, K_COMMIT, launch_commit(c->conf, c->tok, c->canvas_dev, c->committed_dev, B,
                                         cf.canvas_len, -1, c->steps_dev, cf.mask_id, c->stream));
  } else {
    EbMergeArgs m;
    memset(&m, 0, sizeof(m));
    m.T = T; m.n_vblocks = a.n_vblocks;
    m.hm = c->head_m; m.hs = c->head_s; m.hq = c->head_q; m.ha = c->head_a;
    m.inv_temp = c->eb_inv_temp;
    m.H = c->eb_H; m.tok = c->tok; m.max_logit = c->head_max; m.sum = c->eb_sum;
    DG_LAUNCH(c, K_HEAD_MERGE, launch_eb_merge(m, c->stream));
    EbCommitArgs e;
    memset(&e, 0, sizeof(e));
    e.B = B; e.Tc = cf.canvas_len; e.T = T; e.mask_id = cf.mask_id; e.vocab = cf.vocab; e.d = d;
    e.n_vblocks = a.n_vblocks;
    e.H = c->eb_H; e.argmax = c->tok; e.u = c->eb_u; e.hn = c->x; e.embed = c->embed;
    e.head_m = c->head_m; e.head_s = c->head_s; e.max_logit = c->head_max; e.sum = c->eb_sum;
    e.inv_temp = c->eb_inv_temp;
    e.prev_in = c->eb_prev; e.prev_out = c->eb_prev;
    e.state = c->eb_state; e.state_out = c->eb_state;
    e.last_flag = c->eb_last;
    e.bound = kEbBound; e.threshold = kEbStopEntropy;
    e.canvas = c->canvas_dev; e.committed = c->committed_dev; e.stopped = c->eb_stopped;
    e.drawn_out = c->eb_drawn;
    DG_LAUNCH(c, K_COMMIT, launch_eb_commit(e, c->stream));
  }
  c->last_T = T;
  c->last_B = B;
  return DG_OK;
}

void drop_graphs(dg_ctx* c) {
  for (auto& g : c->graphs) cudaGraphExecDestroy(g.second.exec);
  c->graphs.clear();
}

bool graphs_enabled(const dg_ctx* c) {
  const char* e = std::getenv("DG_NO_GRAPH");
  const bool off = e && e[0] && e[0] != '0';
  return !off && !c->prof_on && c->stream != nullptr && c->stream != cudaStreamLegacy &&
         c->stream != cudaStreamPerThread;
}

// One pass: the kernels run from a CUDA graph captured on the second pass of a
// given (batch size, kind) (the first runs directly and sets kernel attributes).
int run_step(dg_ctx* c, int B, int steps_left, bool eb = false) {
  int rc;
  if ((rc = ensure_rope(c, c->layers[0].kv_P)) != DG_OK) return rc;
  if (!eb) DG_CUDA(c, launch_set_int(c->steps_dev, steps_left, c->stream));
  if (!graphs_enabled(c)) return record_step(c, B, eb);
  const int key = 2 * B + (eb ? 1 : 0);
  auto it = c->graphs.find(key);
  if (it == c->graphs.end()) {
    if (!c->warm[key]) {
      c->warm[key] = true;
      return record_step(c, B, eb);
    }
    cudaGraph_t g = nullptr;
    DG_CUDA(c, cudaStreamBeginCapture(c->stream, cudaStreamCaptureModeThreadLocal));
    rc = record_step(c, B, eb);
    const cudaError_t e = cudaStreamEndCapture(c->stream, &g);
    if (rc != DG_OK) {
      if (g) cudaGraphDestroy(g);
      return rc;
    }
    if (e != cudaSuccess) return fail(c, DG_ERR_CUDA, std::string("graph capture: ") + cudaGetErrorString(e));
    dg_ctx::StepGraph sg;
    const cudaError_t e2 = cudaGraphInstantiate(&sg.exec, g, 0);
    cudaGraphDestroy(g);
    if (e2 != cudaSuccess) return fail(c, DG_ERR_CUDA, std::string("graph instantiate: ") + cudaGetErrorString(e2));
    sg.launches = c->launches;
    it = c->graphs.emplace(key, sg).first;
  }
  DG_CUDA(c, cudaGraphLaunch(it->second.exec, c->stream));
  c->launches = it->second.launches;
  c->last_T = B * c->cfg.canvas_len;
  c->last_B = B;
  return DG_OK;
}

// One entropy-bounded pass on c->canvas_dev: temperature and last-pass flag of
// pass `step` of at most `n_max`, the uniforms copied into c->eb_u.
int eb_pass(dg_ctx* c, int B, int step, int n_max, const float* u) {
  const size_t T = (size_t)B * c->cfg.canvas_len;
  const double temp = n_max == 1 ? kEbTempStart
                                 : kEbTempStart + (kEbTempEnd - kEbTempStart) * step / (n_max - 1);
  if (step == 0) DG_CUDA(c, cudaMemsetAsync(c->eb_state, 0, sizeof(int) * B, c->stream));
  DG_CUDA(c, launch_set_float(c->eb_inv_temp, (float)(1.0 / temp), c->stream));
  DG_CUDA(c, launch_set_int(c->eb_last, step == n_max - 1 ? 1 : 0, c->stream));
  DG_CUDA(c, cudaMemcpyAsync(c->eb_u, u, T * 4, cudaMemcpyDefault, c->stream));
  return run_step(c, B, 0, true);
}

int check_eb_args(dg_ctx* c, const void* canvas, int batch, const float* u, int n_max) {
  if (!canvas || !u) return fail(c, DG_ERR_INVALID_ARG, "null canvas or uniforms");
  if (batch < 1 || batch > c->cfg.max_batch) return fail(c, DG_ERR_INVALID_ARG, "batch out of range");
  if (n_max < 1) return fail(c, DG_ERR_INVALID_ARG, "n_max must be >= 1");
  if (!c->weights_ready) return fail(c, DG_ERR_BAD_STATE, "weights not initialised");
  if (c->cfg.canvas_len > 256 || c->cfg.d_model % 8)
    return fail(c, DG_ERR_UNSUPPORTED, "entropy-bounded passes need canvas_len <= 256");
  return check_prompt_state(c, batch);
}

int read_device_error(dg_ctx* c) {
  int h = 0;
  DG_CUDA(c, cudaMemcpyAsync(&h, c->err_dev, sizeof(int), cudaMemcpyDeviceToHost, c->stream));
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  if (h != 0) {
    DG_CUDA(c, cudaMemsetAsync(c->err_dev, 0, sizeof(int), c->stream));
    DG_CUDA(c, cudaStreamSynchronize(c->stream));
    if (h == kErrTimeout) return fail(c, DG_ERR_TIMEOUT, "a bounded device wait gave up");
    return fail(c, DG_ERR_DEVICE_FAULT, "a kernel flagged an out-of-range index");
  }
  return DG_OK;
}

// Point every layer's prompt K/V at the library's own cache: batch B, the
// positions encoded so far (ctx_len), rows max_context apart.
int use_own_cache(dg_ctx* c, int B) {
  const dg_config& cf = c->cfg;
  for (auto& L : c->layers) {
    if (L.kp != L.own_k || L.kv_batch != B || L.kv_P != c->ctx_len) drop_graphs(c);
    if (L.kp != L.own_k || L.kv_batch != B) {
      const uint64_t rows = (uint64_t)B * cf.n_kv_heads * cf.max_context;
      if (!make_tmap_2d(&L.m_kp, L.own_k, cf.head_dim, rows, 64) ||
          !make_tmap_2d(&L.m_vp, L.own_v, cf.head_dim, rows, 64))
        return fail(c, DG_ERR_CUDA, "tensor map for the context K/V failed");
    }
    L.kp = L.own_k;
    L.vp = L.own_v;
    L.kv_batch = B;
    L.kv_P = c->ctx_len;
    L.kv_stride = cf.max_context;
  }
  return DG_OK;
}

// The causal encoder over n tokens per sequence (device or host int32 [B][n],
// row stride ld), in chunks of up to Tmax / B tokens (the rows a pass over
// max_batch canvases holds): each chunk's keys and values are appended to the
// own cache after the positions already held.  Every chunk reads all the
// layers' weights once, so the longer the chunk the fewer weight bytes a token.
int encode_tokens(dg_ctx* c, const int32_t* tokens, int B, int n, int ld) {
  const dg_config& cf = c->cfg;
  const int chunk = std::max(1, c->Tmax / B);
  int rc;
  for (int o = 0; o < n; o += chunk) {
    const int m = std::min(chunk, n - o);
    if ((rc = use_own_cache(c, B)) != DG_OK) return rc;
    if ((rc = ensure_rope(c, c->ctx_len)) != DG_OK) return rc;
    DG_CUDA(c, cudaMemcpy2DAsync(c->canvas_dev, (size_t)m * 4, tokens + o, (size_t)ld * 4,
                                 (size_t)m * 4, B, cudaMemcpyDefault, c->stream));
    DG_LAUNCH(c, K_EMBED, launch_embed_norm(c->canvas_dev, c->embed, nullptr, cf.vocab, B * m,
                                            cf.d_model, c->layers[0].ln_in, cf.rms_eps, c->h,
                                            c->x, c->err_dev, c->stream));
    for (int l = 0; l < cf.n_layers; ++l) {
      const float* w_next = (l + 1 < cf.n_layers) ? c->layers[l + 1].ln_in : c->ln_final;
      if ((rc = run_layer(c, l, B, w_next, m, true)) != DG_OK) return rc;
    }
    c->ctx_len += m;
    c->ctx_batch = B;
  }
  return DG_OK;
}

int check_context_args(dg_ctx* c, int batch, int n) {
  if (c->cfg.max_context < 1)
    return fail(c, DG_ERR_BAD_STATE, "the context needs dg_config.max_context > 0");
  if (!c->weights_ready) return fail(c, DG_ERR_BAD_STATE, "weights not initialised");
  if (batch < 1 || batch > c->cfg.max_batch) return fail(c, DG_ERR_INVALID_ARG, "batch out of range");
  if (c->ctx_len > 0 && batch != c->ctx_batch)
    return fail(c, DG_ERR_INVALID_ARG, "batch differs from the batch of the encoded context");
  if (n < 0 || (long long)c->ctx_len + n > c->cfg.max_context)
    return fail(c, DG_ERR_INVALID_ARG, "the context would exceed max_context");
  return DG_OK;
}

}  // namespace

extern "C" {

int dg_create(const dg_config* cfg, void* cuda_stream, dg_ctx** out) {
  if (!cfg || !out) return fail(nullptr, DG_ERR_INVALID_ARG, "null argument");
  const std::string why = check_config(*cfg);
  if (!why.empty()) return fail(nullptr, DG_ERR_INVALID_ARG, why);
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    return fail(nullptr, DG_ERR_CUDA, "no CUDA device");
  }
  dg_ctx* c = new (std::nothrow) dg_ctx();
  if (!c) return fail(nullptr, DG_ERR_OOM, "host allocation failed");
  c->cfg = *cfg;
  c->stream = static_cast<cudaStream_t>(cuda_stream);
  cudaGetDevice(&c->device);
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, c->device) != cudaSuccess) {
    delete c;
    return fail(nullptr, DG_ERR_CUDA, "cudaGetDeviceProperties failed");
  }
  if (prop.major != 10) {
    delete c;
    return fail(nullptr, DG_ERR_UNSUPPORTED, "needs an sm_100 (B200) device");
  }
  c->num_sms = prop.multiProcessorCount;
  {
    const char* e = std::getenv("DG_CTA_PAIR");
    c->pair_clusters = (e && e[0] && e[0] != '0') ? gemm_pair_max_clusters() : 0;
    const char* fr = std::getenv("DG_FUSED_ROUTER");
    c->fused_router = fr && fr[0] && fr[0] != '0';
    const char* cm = std::getenv("DG_ATTN_CLUSTER_MERGE");
    c->attn_cluster_merge = cm && cm[0] && cm[0] != '0';
    // whether each cluster size fits is asked once here, outside any graph capture
    if (c->attn_cluster_merge)
      for (int n = 1; n <= 8; ++n) attn_tc_fused_ok(c->cfg.head_dim, n);
  }
  const dg_config& cf = c->cfg;
  const int d = cf.d_model, F = cf.d_ff, dh = cf.head_dim, E = cf.n_experts, k = cf.top_k;
  const int Hq = cf.n_q_heads, Hkv = cf.n_kv_heads;
  c->Tmax = cf.max_batch * cf.canvas_len;
  c->dense_box = std::min(256, (c->Tmax + 31) / 32 * 32);
  c->NQKV = (Hq + 2 * Hkv) * dh;
  c->G = E + 1;
  const size_t T = c->Tmax, V = cf.vocab;
  // Row counts of TMA-read buffers are padded so that no box is taller than its tensor.
  const size_t Tp = std::max<size_t>(128, (T + 127) / 128 * 128);
  const size_t Er = (size_t)std::max(E, 128);
  bool ok = true;
  ok &= alloc_n(c, &c->embed, V * d);
  ok &= alloc_n(c, &c->ln_final, d);
  c->layers.resize(cf.n_layers);
  for (auto& L : c->layers) {
    ok &= alloc_n(c, &L.wqkv, (size_t)c->NQKV * d);
    ok &= alloc_n(c, &L.wo, (size_t)d * Hq * dh);
    ok &= alloc_n(c, &L.wr, Er * d);
    if (cf.max_context > 0) {
      const size_t cap = (size_t)cf.max_batch * Hkv * cf.max_context * dh;
      ok &= alloc_n(c, &L.own_k, cap);
      ok &= alloc_n(c, &L.own_v, cap);
    }
    ok &= alloc_n(c, &L.wgu, (size_t)c->G * 2 * F * d);
    ok &= alloc_n(c, &L.wd, (size_t)c->G * d * F);
    if (cf.expert_dtype == DG_DTYPE_FP8_E4M3) {
      ok &= alloc_n(c, &L.wgu8, (size_t)c->G * 2 * F * d);
      ok &= alloc_n(c, &L.wd8, (size_t)c->G * d * F);
      ok &= alloc_n(c, &L.sgu, (size_t)c->G * 2 * F);
      ok &= alloc_n(c, &L.sd8, (size_t)c->G * d);
    }
    ok &= alloc_n(c, &L.ln_in, d);
    ok &= alloc_n(c, &L.ln_post, d);
    ok &= alloc_n(c, &L.ln_ff, d);
    if (!ok) break;
  }
  const size_t rows_moe = std::max<size_t>(128, (size_t)(k + 1) * T);
  c->part_elems = std::max({(size_t)kMaxSplits * T * c->NQKV, (size_t)kMaxSplits * T * d,
                            (size_t)kMaxSplits * T * E});
  if (ok) {
    ok &= alloc_n(c, &c->h, T * d);
    ok &= alloc_n(c, &c->x, Tp * d);
    ok &= alloc_n(c, &c->part, c->part_elems);
    ok &= alloc_n(c, &c->q, std::max<size_t>(T * Hq, 128) * dh);
    ok &= alloc_n(c, &c->kc, std::max<size_t>(T * Hkv, 64) * dh);
    ok &= alloc_n(c, &c->vc, std::max<size_t>(T * Hkv, 64) * dh);
    ok &= alloc_n(c, &c->attn_po, (size_t)kMaxAttnChunks * T * Hq * dh);
    ok &= alloc_n(c, &c->attn_ml, (size_t)kMaxAttnChunks * T * Hq * 2);
    ok &= alloc_n(c, &c->attn_o, Tp * Hq * dh);
    ok &= alloc_n(c, &c->xperm, rows_moe * d);
    ok &= alloc_n(c, &c->router_logits, T * E);
    ok &= alloc_n(c, &c->idx, T * k);
    ok &= alloc_n(c, &c->w, T * k);
    ok &= alloc_n(c, &c->bitmap, (size_t)E * ((T + 31) / 32));
    ok &= alloc_n(c, &c->router_counter, 4);
    // every expert chunk of a layer: the shared group's plus the routed groups'
    c->chunk_rows = kGroupedTile;
    const size_t cr = (size_t)c->chunk_rows;
    c->n_chunk_ready = (int)((T + cr - 1) / cr + ((size_t)k * T + cr - 1) / cr + E);
    ok &= alloc_n(c, &c->chunk_ready, (size_t)c->n_chunk_ready);
    ok &= alloc_n(c, &c->chunk_order, (size_t)c->n_chunk_ready);
    ok &= alloc_n(c, &c->tile_counters, 2);
    ok &= alloc_n(c, &c->steps_dev, 4);
    ok &= alloc_n(c, &c->offsets_r, E + 1);
    ok &= alloc_n(c, &c->offsets_g, E + 2);
    ok &= alloc_n(c, &c->chunk_prefix, E + 2);
    ok &= alloc_n(c, &c->perm, T * k);
    ok &= alloc_n(c, &c->inv, T * k);
    ok &= alloc_n(c, &c->H, rows_moe * F);
    ok &= alloc_n(c, &c->Y, rows_moe * d);
    const size_t nvb = (V + 255) / 256;
    ok &= alloc_n(c, &c->head_m, nvb * T);
    ok &= alloc_n(c, &c->head_s, nvb * T);
    ok &= alloc_n(c, &c->head_a, nvb * T);
    ok &= alloc_n(c, &c->conf, T);
    ok &= alloc_n(c, &c->head_max, T);
    ok &= alloc_n(c, &c->head_q, ((V + 255) / 256) * T);
    ok &= alloc_n(c, &c->eb_H, T);
    ok &= alloc_n(c, &c->eb_sum, T);
    ok &= alloc_n(c, &c->eb_u, T);
    ok &= alloc_n(c, &c->eb_prev, T);
    ok &= alloc_n(c, &c->eb_drawn, T);
    ok &= alloc_n(c, &c->eb_state, cf.max_batch);
    ok &= alloc_n(c, &c->eb_stopped, cf.max_batch);
    ok &= alloc_n(c, &c->eb_inv_temp, 4);
    ok &= alloc_n(c, &c->eb_last, 4);
    ok &= alloc_n(c, &c->tok, T);
    ok &= alloc_n(c, &c->canvas_dev, T);
    if (cf.max_context > 0) ok &= alloc_n(c, &c->gen_canvas, T);
    ok &= alloc_n(c, &c->committed_dev, T);
    ok &= alloc_n(c, &c->err_dev, 4);
    ok &= alloc_n(c, &c->expert_active, cf.n_layers);
    ok &= alloc_n(c, &c->rope_cos, (size_t)c->Tmax * dh / 2);
    ok &= alloc_n(c, &c->rope_sin, (size_t)c->Tmax * dh / 2);
    ok &= alloc_n(c, &c->router_bias, E);
  }
  if (!ok) {
    const size_t have = c->bytes;
    free_all(c);
    delete c;
    return fail(nullptr, DG_ERR_OOM,
                "device allocation failed or passed alloc_limit_bytes (after " +
                    std::to_string(have) + " bytes)");
  }
  // zero the scratch that kernels accumulate into or read before writing
  cudaMemset(c->bitmap, 0, (size_t)E * ((T + 31) / 32) * 4);
  cudaMemset(c->router_counter, 0, 16);
  cudaMemset(c->chunk_ready, 0, sizeof(int) * (size_t)c->n_chunk_ready);
  cudaMemset(c->chunk_order, 0, sizeof(int) * (size_t)c->n_chunk_ready);
  cudaMemset(c->tile_counters, 0, sizeof(int) * 2);
  cudaMemset(c->err_dev, 0, 16);
  cudaMemset(c->eb_state, 0, sizeof(int) * cf.max_batch);
  cudaMemset(c->expert_active, 0, sizeof(int) * cf.n_layers);
  cudaMemset(c->xperm, 0, rows_moe * d * 2);
  cudaMemset(c->H, 0, rows_moe * F * 2);
  cudaMemset(c->x, 0, Tp * d * 2);
  // rows past T read by attention tiles must be finite (a masked key still multiplies V)
  cudaMemset(c->q, 0, std::max<size_t>(T * Hq, 128) * dh * 2);
  cudaMemset(c->kc, 0, std::max<size_t>(T * Hkv, 64) * dh * 2);
  cudaMemset(c->vc, 0, std::max<size_t>(T * Hkv, 64) * dh * 2);
  cudaMemset(c->attn_o, 0, Tp * Hq * dh * 2);
  for (auto& L : c->layers) cudaMemset(L.wr, 0, Er * d * 2);
  // tensor maps (weights: A operands, 128-row boxes; activations: B operands, 32-row boxes)
  ok = make_tmap_2d(&c->m_embed, c->embed, d, V, 256);
  for (auto& L : c->layers) {
    ok &= make_tmap_2d(&L.m_qkv, L.wqkv, d, c->NQKV, 128);
    ok &= make_tmap_2d(&L.m_o, L.wo, (uint64_t)Hq * dh, d, 128);
    ok &= make_tmap_2d(&L.m_r, L.wr, d, Er, 128);
    ok &= make_tmap_3d(&L.m_gu, L.wgu, d, 2 * F, c->G, 128);
    ok &= make_tmap_3d(&L.m_d, L.wd, F, d, c->G, 128);
    if (L.wgu8) {
      ok &= make_tmap_3d_u8(&L.m_gu8, L.wgu8, d, 2 * F, c->G);
      ok &= make_tmap_3d_u8(&L.m_d8, L.wd8, F, d, c->G);
    }
  }
  ok &= make_tmap_2d(&c->m_x_b, c->x, d, Tp, c->dense_box);
  ok &= make_tmap_2d(&c->m_x_a, c->x, d, Tp, 128);
  ok &= make_tmap_2d(&c->m_attn_o_b, c->attn_o, (uint64_t)Hq * dh, Tp, c->dense_box);
  ok &= make_tmap_2d(&c->m_x_bh, c->x, d, Tp, c->dense_box / 2);
  ok &= make_tmap_2d(&c->m_attn_o_bh, c->attn_o, (uint64_t)Hq * dh, Tp, c->dense_box / 2);
  ok &= make_tmap_2d(&c->m_xperm_b, c->xperm, d, rows_moe, kGroupedBox);
  ok &= make_tmap_2d(&c->m_x2_b, c->xperm, d, rows_moe, c->dense_box);
  ok &= make_tmap_2d(&c->m_H_b, c->H, F, rows_moe, kGroupedBox);
  ok &= make_tmap_out_f32(&c->m_Y_out, c->Y, d, rows_moe, 1);
  ok &= make_tmap_h_store(&c->m_H_out, c->H, F, rows_moe);
  ok &= make_tmap_2d(&c->m_q, c->q, dh, std::max<size_t>(T * Hq, 128), 128);
  ok &= make_tmap_f32_sw128(&c->m_attn_po, c->attn_po, dh, (uint64_t)kMaxAttnChunks * T * Hq);
  ok &= make_tmap_2d(&c->m_kc, c->kc, dh, std::max<size_t>(T * Hkv, 64), 64);
  ok &= make_tmap_2d(&c->m_vc, c->vc, dh, std::max<size_t>(T * Hkv, 64), 64);
  if (cudaDeviceSynchronize() != cudaSuccess || !ok) {
    cudaGetLastError();
    free_all(c);
    delete c;
    return fail(nullptr, DG_ERR_CUDA, "tensor map creation or initial memset failed");
  }
  *out = c;
  return DG_OK;
}

int dg_init_weights(dg_ctx* c, uint64_t seed) {
  if (!c) return DG_ERR_INVALID_ARG;
  const dg_config& cf = c->cfg;
  const int d = cf.d_model, F = cf.d_ff, dh = cf.head_dim, E = cf.n_experts;
  const int Hq = cf.n_q_heads, Hkv = cf.n_kv_heads;
  const float scale = (float)(cf.weight_std * std::sqrt(3.0) / 65536.0);
  auto key = [&](unsigned long long tid) { return stream_key_host(seed, tid); };
  auto ltid = [](int l, int kind) { return 64ull * (unsigned long long)(l + 1) + (unsigned)kind; };
  InitArgs a;
  memset(&a, 0, sizeof(a));
  a.scale = scale;
  a.layout = INIT_PLAIN;
  a.dst = c->embed;
  a.n_elems = (long long)cf.vocab * d;
  a.key0 = key(1);
  DG_CUDA(c, launch_init(a, c->stream));
  DG_CUDA(c, launch_fill_f32(c->ln_final, d, 1.0f, c->stream));
  for (int l = 0; l < cf.n_layers; ++l) {
    Layer& L = c->layers[l];
    memset(&a, 0, sizeof(a));
    a.scale = scale;
    a.layout = INIT_QKV; a.dst = L.wqkv; a.n_elems = (long long)c->NQKV * d;
    a.key0 = key(ltid(l, 0)); a.key1 = key(ltid(l, 1)); a.key2 = key(ltid(l, 2));
    a.rows_a = Hq * dh; a.rows_b = Hkv * dh; a.cols = d;
    DG_CUDA(c, launch_init(a, c->stream));
    a.layout = INIT_PLAIN; a.dst = L.wo; a.n_elems = (long long)d * Hq * dh; a.key0 = key(ltid(l, 3));
    DG_CUDA(c, launch_init(a, c->stream));
    a.dst = L.wr; a.n_elems = (long long)E * d; a.key0 = key(ltid(l, 4));
    DG_CUDA(c, launch_init(a, c->stream));
    a.layout = INIT_GATEUP; a.dst = L.wgu; a.n_elems = (long long)c->G * 2 * F * d;
    a.key0 = key(ltid(l, 5)); a.key1 = key(ltid(l, 6)); a.key2 = key(ltid(l, 8)); a.key3 = key(ltid(l, 9));
    a.F = F; a.d = d; a.E = E;
    DG_CUDA(c, launch_init(a, c->stream));
    a.layout = INIT_DOWN; a.dst = L.wd; a.n_elems = (long long)c->G * d * F;
    a.key0 = key(ltid(l, 7)); a.key1 = key(ltid(l, 10));
    DG_CUDA(c, launch_init(a, c->stream));
    DG_CUDA(c, launch_fill_f32(L.ln_in, d, 1.0f, c->stream));
    DG_CUDA(c, launch_fill_f32(L.ln_post, d, 1.0f, c->stream));
    DG_CUDA(c, launch_fill_f32(L.ln_ff, d, 1.0f, c->stream));
    int rc = quantize_layer(c, L);
    if (rc != DG_OK) return rc;
  }
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  c->weights_ready = true;
  return DG_OK;
}

int dg_set_prompt_kv(dg_ctx* c, int layer, const void* k, const void* v, int batch, int n_prompt) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (layer < 0 || layer >= c->cfg.n_layers) return fail(c, DG_ERR_INVALID_ARG, "layer out of range");
  if (!k || !v) return fail(c, DG_ERR_INVALID_ARG, "null prompt K/V");
  if (batch < 1 || batch > c->cfg.max_batch) return fail(c, DG_ERR_INVALID_ARG, "batch out of range");
  if (n_prompt < 1 || n_prompt > c->cfg.max_prompt)
    return fail(c, DG_ERR_INVALID_ARG, "n_prompt out of range");
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15)
    return fail(c, DG_ERR_INVALID_ARG, "prompt K/V must be 16-byte aligned");
  Layer& L = c->layers[layer];
  if (L.kp != k || L.vp != v || L.kv_batch != batch || L.kv_P != n_prompt) {
    drop_graphs(c);
    const uint64_t rows = (uint64_t)batch * c->cfg.n_kv_heads * n_prompt;
    if (!make_tmap_2d(&L.m_kp, k, c->cfg.head_dim, rows, 64) ||
        !make_tmap_2d(&L.m_vp, v, c->cfg.head_dim, rows, 64))
      return fail(c, DG_ERR_CUDA, "tensor map for the prompt K/V failed");
  }
  L.kp = static_cast<const bf16*>(k);
  L.vp = static_cast<const bf16*>(v);
  L.kv_batch = batch;
  L.kv_P = n_prompt;
  L.kv_stride = n_prompt;
  return DG_OK;
}

int dg_encode(dg_ctx* c, const int32_t* tokens, int batch, int n) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (!tokens) return fail(c, DG_ERR_INVALID_ARG, "null tokens");
  if (n < 1) return fail(c, DG_ERR_INVALID_ARG, "n must be >= 1");
  int rc = check_context_args(c, batch, n);
  if (rc != DG_OK) return rc;
  if ((rc = encode_tokens(c, tokens, batch, n, n)) != DG_OK) return rc;
  if ((rc = use_own_cache(c, batch)) != DG_OK) return rc;
  return read_device_error(c);
}

int dg_reset_context(dg_ctx* c) {
  if (!c) return DG_ERR_INVALID_ARG;
  c->ctx_len = 0;
  c->ctx_batch = 0;
  return DG_OK;
}

int dg_context_length(dg_ctx* c, int* n_out) {
  if (!c || !n_out) return DG_ERR_INVALID_ARG;
  *n_out = c->ctx_len;
  return DG_OK;
}

int dg_context_kv(dg_ctx* c, int layer, void* k_out, void* v_out) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (layer < 0 || layer >= c->cfg.n_layers) return fail(c, DG_ERR_INVALID_ARG, "layer out of range");
  if (!k_out || !v_out) return fail(c, DG_ERR_INVALID_ARG, "null output");
  if (c->cfg.max_context < 1 || c->ctx_len == 0)
    return fail(c, DG_ERR_BAD_STATE, "no encoded context");
  const dg_config& cf = c->cfg;
  const Layer& L = c->layers[layer];
  const size_t row = (size_t)cf.head_dim * 2;
  const int seqs = c->ctx_batch * cf.n_kv_heads;
  DG_CUDA(c, cudaMemcpy2DAsync(k_out, c->ctx_len * row, L.own_k, (size_t)cf.max_context * row,
                               c->ctx_len * row, seqs, cudaMemcpyDefault, c->stream));
  DG_CUDA(c, cudaMemcpy2DAsync(v_out, c->ctx_len * row, L.own_v, (size_t)cf.max_context * row,
                               c->ctx_len * row, seqs, cudaMemcpyDefault, c->stream));
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  return DG_OK;
}

int dg_set_router_bias(dg_ctx* c, const float* bias) {
  if (!c) return DG_ERR_INVALID_ARG;
  drop_graphs(c);
  if (!bias) { c->has_bias = false; return DG_OK; }
  DG_CUDA(c, cudaMemcpyAsync(c->router_bias, bias, sizeof(float) * c->cfg.n_experts,
                             cudaMemcpyDefault, c->stream));
  c->has_bias = true;
  return DG_OK;
}

int dg_canvas_step(dg_ctx* c, int32_t* canvas, int batch, int steps_left, float* conf_out,
                   uint8_t* committed_out) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (!canvas) return fail(c, DG_ERR_INVALID_ARG, "null canvas");
  if (batch < 1 || batch > c->cfg.max_batch) return fail(c, DG_ERR_INVALID_ARG, "batch out of range");
  if (steps_left < 1) return fail(c, DG_ERR_INVALID_ARG, "steps_left must be >= 1");
  if (!c->weights_ready) return fail(c, DG_ERR_BAD_STATE, "weights not initialised");
  int rc = check_prompt_state(c, batch);
  if (rc != DG_OK) return rc;
  const size_t T = (size_t)batch * c->cfg.canvas_len;
  DG_CUDA(c, cudaMemcpyAsync(c->canvas_dev, canvas, T * 4, cudaMemcpyDefault, c->stream));
  if ((rc = run_step(c, batch, steps_left)) != DG_OK) return rc;
  DG_CUDA(c, cudaMemcpyAsync(canvas, c->canvas_dev, T * 4, cudaMemcpyDefault, c->stream));
  if (conf_out) DG_CUDA(c, cudaMemcpyAsync(conf_out, c->conf, T * 4, cudaMemcpyDefault, c->stream));
  if (committed_out)
    DG_CUDA(c, cudaMemcpyAsync(committed_out, c->committed_dev, T, cudaMemcpyDefault, c->stream));
  return DG_OK;
}

int dg_canvas_step_host(dg_ctx* c, int32_t* canvas_host, int batch, int steps_left,
                        float* conf_host, uint8_t* committed_host) {
  if (!c) return DG_ERR_INVALID_ARG;
  int rc = dg_canvas_step(c, canvas_host, batch, steps_left, conf_host, committed_host);
  if (rc != DG_OK) return rc;
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  return read_device_error(c);
}

int dg_denoise_block(dg_ctx* c, int32_t* canvas, int batch, int n_steps) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (n_steps < 1) return fail(c, DG_ERR_INVALID_ARG, "n_steps must be >= 1");
  if (!canvas) return fail(c, DG_ERR_INVALID_ARG, "null canvas");
  if (batch < 1 || batch > c->cfg.max_batch) return fail(c, DG_ERR_INVALID_ARG, "batch out of range");
  if (!c->weights_ready) return fail(c, DG_ERR_BAD_STATE, "weights not initialised");
  int rc = check_prompt_state(c, batch);
  if (rc != DG_OK) return rc;
  const size_t T = (size_t)batch * c->cfg.canvas_len;
  DG_CUDA(c, cudaMemcpyAsync(c->canvas_dev, canvas, T * 4, cudaMemcpyDefault, c->stream));
  for (int s = 0; s < n_steps; ++s)
    if ((rc = run_step(c, batch, n_steps - s)) != DG_OK) return rc;
  DG_CUDA(c, cudaMemcpyAsync(canvas, c->canvas_dev, T * 4, cudaMemcpyDefault, c->stream));
  return read_device_error(c);
}

int dg_generate(dg_ctx* c, const int32_t* prompt, int batch, int n_prompt, int n_blocks,
                int n_steps, int32_t* out) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (!prompt || !out) return fail(c, DG_ERR_INVALID_ARG, "null prompt or output");
  if (n_prompt < 1 || n_blocks < 1 || n_steps < 1)
    return fail(c, DG_ERR_INVALID_ARG, "n_prompt, n_blocks and n_steps must be >= 1");
  const dg_config& cf = c->cfg;
  const int Tc = cf.canvas_len;
  dg_reset_context(c);
  int rc = check_context_args(c, batch, n_prompt + n_blocks * Tc);
  if (rc != DG_OK) return rc;
  if ((rc = encode_tokens(c, prompt, batch, n_prompt, n_prompt)) != DG_OK) return rc;
  const std::vector<int32_t> mask((size_t)batch * Tc, cf.mask_id);
  const size_t row_out = (size_t)n_blocks * Tc * 4;
  for (int blk = 0; blk < n_blocks; ++blk) {
    // an all-mask canvas denoised against the context, then encoded onto it
    if ((rc = use_own_cache(c, batch)) != DG_OK) return rc;
    DG_CUDA(c, cudaMemcpyAsync(c->gen_canvas, mask.data(), mask.size() * 4, cudaMemcpyHostToDevice,
                               c->stream));
    if ((rc = dg_denoise_block(c, c->gen_canvas, batch, n_steps)) != DG_OK) return rc;
    DG_CUDA(c, cudaMemcpy2DAsync(out + (size_t)blk * Tc, row_out, c->gen_canvas, (size_t)Tc * 4,
                                 (size_t)Tc * 4, batch, cudaMemcpyDefault, c->stream));
    if ((rc = encode_tokens(c, c->gen_canvas, batch, Tc, Tc)) != DG_OK) return rc;
  }
  if ((rc = use_own_cache(c, batch)) != DG_OK) return rc;
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  return read_device_error(c);
}

int dg_eb_step(dg_ctx* c, int32_t* canvas, int batch, int step, int n_max, const float* u,
               float* entropy_out, uint8_t* committed_out, uint8_t* stopped_out) {
  if (!c) return DG_ERR_INVALID_ARG;
  int rc = check_eb_args(c, canvas, batch, u, n_max);
  if (rc != DG_OK) return rc;
  if (step < 0 || step >= n_max) return fail(c, DG_ERR_INVALID_ARG, "step must be in [0, n_max)");
  const size_t T = (size_t)batch * c->cfg.canvas_len;
  DG_CUDA(c, cudaMemcpyAsync(c->canvas_dev, canvas, T * 4, cudaMemcpyDefault, c->stream));
  if ((rc = eb_pass(c, batch, step, n_max, u)) != DG_OK) return rc;
  DG_CUDA(c, cudaMemcpyAsync(canvas, c->canvas_dev, T * 4, cudaMemcpyDefault, c->stream));
  if (entropy_out)
    DG_CUDA(c, cudaMemcpyAsync(entropy_out, c->eb_H, T * 4, cudaMemcpyDefault, c->stream));
  if (committed_out)
    DG_CUDA(c, cudaMemcpyAsync(committed_out, c->committed_dev, T, cudaMemcpyDefault, c->stream));
  if (stopped_out)
    DG_CUDA(c, cudaMemcpyAsync(stopped_out, c->eb_stopped, batch, cudaMemcpyDefault, c->stream));
  return DG_OK;
}

int dg_eb_denoise_block(dg_ctx* c, int32_t* canvas, int batch, int n_max, const float* u,
                        int* passes_out) {
  if (!c) return DG_ERR_INVALID_ARG;
  int rc = check_eb_args(c, canvas, batch, u, n_max);
  if (rc != DG_OK) return rc;
  const size_t T = (size_t)batch * c->cfg.canvas_len;
  std::vector<int> state(batch, 0), passes(batch, 0);
  DG_CUDA(c, cudaMemcpyAsync(c->canvas_dev, canvas, T * 4, cudaMemcpyDefault, c->stream));
  for (int s = 0; s < n_max; ++s) {
    if ((rc = eb_pass(c, batch, s, n_max, u + (size_t)s * T)) != DG_OK) return rc;
    for (int b = 0; b < batch; ++b) passes[b] += (state[b] & 2) ? 0 : 1;
    DG_CUDA(c, cudaMemcpyAsync(state.data(), c->eb_state, sizeof(int) * batch,
                               cudaMemcpyDeviceToHost, c->stream));
    DG_CUDA(c, cudaStreamSynchronize(c->stream));
    bool all_done = true;
    for (int b = 0; b < batch; ++b) all_done = all_done && (state[b] & 2);
    if (all_done) break;
  }
  DG_CUDA(c, cudaMemcpyAsync(canvas, c->canvas_dev, T * 4, cudaMemcpyDefault, c->stream));
  if (passes_out) std::copy(passes.begin(), passes.end(), passes_out);
  return read_device_error(c);
}

int dg_eb_commit(dg_ctx* c, const float* entropy, const int32_t* argmax, const int32_t* drawn,
                 const int32_t* prev_argmax, int32_t* canvas, int batch, int last,
                 uint8_t* committed_out, uint8_t* stopped_out) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (!entropy || !argmax || !drawn || !canvas) return fail(c, DG_ERR_INVALID_ARG, "null argument");
  if (batch < 1 || batch > c->cfg.max_batch) return fail(c, DG_ERR_INVALID_ARG, "batch out of range");
  if (c->cfg.canvas_len > 256) return fail(c, DG_ERR_UNSUPPORTED, "canvas_len must be <= 256");
  EbCommitArgs e;
  memset(&e, 0, sizeof(e));
  e.B = batch; e.Tc = c->cfg.canvas_len; e.T = batch * c->cfg.canvas_len;
  e.mask_id = c->cfg.mask_id; e.vocab = c->cfg.vocab; e.d = c->cfg.d_model;
  e.H = entropy; e.argmax = argmax; e.drawn_in = drawn; e.prev_in = prev_argmax;
  e.last = last ? 1 : 0;
  e.bound = kEbBound; e.threshold = kEbStopEntropy;
  e.canvas = canvas; e.committed = committed_out; e.stopped = stopped_out;
  DG_CUDA(c, launch_eb_commit(e, c->stream));
  return DG_OK;
}

int dg_layer_forward(dg_ctx* c, int layer, const void* x_in, void* x_out, int n_rows) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (layer < 0 || layer >= c->cfg.n_layers) return fail(c, DG_ERR_INVALID_ARG, "layer out of range");
  if (!x_in || !x_out) return fail(c, DG_ERR_INVALID_ARG, "null hidden-state pointer");
  if (!c->weights_ready) return fail(c, DG_ERR_BAD_STATE, "weights not initialised");
  const Layer& L = c->layers[layer];
  if (!L.kp) return fail(c, DG_ERR_BAD_STATE, "prompt KV not set for this layer");
  if (n_rows != L.kv_batch * c->cfg.canvas_len)
    return fail(c, DG_ERR_INVALID_ARG, "n_rows must equal batch * canvas_len of the prompt KV");
  const int B = L.kv_batch, d = c->cfg.d_model;
  int rc;
  c->launches = 0;
  if ((rc = ensure_rope(c, L.kv_P)) != DG_OK) return rc;
  DG_LAUNCH(c, K_EMBED, launch_embed_norm(nullptr, nullptr, static_cast<const bf16*>(x_in), c->cfg.vocab,
                                 n_rows, d, L.ln_in, c->cfg.rms_eps, c->h, c->x, c->err_dev,
                                 c->stream));
  if ((rc = run_layer(c, layer, B, nullptr, c->cfg.canvas_len, false)) != DG_OK) return rc;
  DG_CUDA(c, cudaMemcpyAsync(x_out, c->x, (size_t)n_rows * d * 2, cudaMemcpyDeviceToDevice,
                             c->stream));
  c->last_T = n_rows;
  c->last_B = B;
  return DG_OK;
}

int dg_router_topk(dg_ctx* c, const float* logits, int n_rows, int32_t* idx, float* w,
                   int32_t* offsets, int32_t* perm) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (!logits || !idx || !w || !offsets || !perm) return fail(c, DG_ERR_INVALID_ARG, "null argument");
  if (n_rows < 1 || n_rows > c->Tmax) return fail(c, DG_ERR_INVALID_ARG, "n_rows out of range");
  if (reinterpret_cast<uintptr_t>(logits) & 15)
    return fail(c, DG_ERR_INVALID_ARG, "logits must be 16-byte aligned");
  RouterArgs ra;
  memset(&ra, 0, sizeof(ra));
  ra.logits_in = logits; ra.splits = 1;
  ra.T = n_rows; ra.E = c->cfg.n_experts; ra.k = c->cfg.top_k; ra.n_shared = 0;
  ra.n_tile = kGroupedTile;
  ra.idx = idx; ra.w = w; ra.bitmap = c->bitmap; ra.counter = c->router_counter;
  ra.offsets_r = offsets; ra.perm = perm; ra.inv = c->inv; ra.err = c->err_dev;
  DG_CUDA(c, launch_router(ra, c->stream));
  return DG_OK;
}

int dg_commit(dg_ctx* c, const float* conf, int32_t* canvas, int batch, int steps_left,
              const int32_t* cand_tok, uint8_t* committed_out) {
  if (!c) return DG_ERR_INVALID_ARG;
  if (!conf || !canvas || !cand_tok) return fail(c, DG_ERR_INVALID_ARG, "null argument");
  if (batch < 1 || batch > c->cfg.max_batch) return fail(c, DG_ERR_INVALID_ARG, "batch out of range");
  if (steps_left < 1) return fail(c, DG_ERR_INVALID_ARG, "steps_left must be >= 1");
  DG_CUDA(c, launch_commit(conf, cand_tok, canvas, committed_out, batch, c->cfg.canvas_len,
                           steps_left, nullptr, c->cfg.mask_id, c->stream));
  return DG_OK;
}

int dg_load_weights(dg_ctx* c, const char* name, const void* src, size_t bytes) {
  if (!c || !name || !src) return DG_ERR_INVALID_ARG;
  if (!c->weights_ready) return fail(c, DG_ERR_BAD_STATE, "weights not initialised");
  const dg_config& cf = c->cfg;
  const size_t d = cf.d_model, E = cf.n_experts, F = cf.d_ff, V = cf.vocab;
  const size_t dh = cf.head_dim, Hq = cf.n_q_heads, Hkv = cf.n_kv_heads;
  const std::string s(name);
  // one contiguous destination, or rows of one bf16 matrix with a row pitch
  void* dst = nullptr;
  size_t n = 0, rows = 0, row_bytes = 0, pitch = 0;
  Layer* requant_layer = nullptr;
  if (s == "embed") { dst = c->embed; n = V * d * 2; }
  else if (s == "ln_final") { dst = c->ln_final; n = d * 4; }
  else {
    const size_t colon = s.find(':');
    if (colon == std::string::npos) return fail(c, DG_ERR_INVALID_ARG, "unknown tensor name");
    const std::string base = s.substr(0, colon);
    const int l = std::atoi(s.c_str() + colon + 1);
    if (l < 0 || l >= cf.n_layers) return fail(c, DG_ERR_INVALID_ARG, "layer out of range");
    Layer& L = c->layers[l];
    bf16* gu = L.wgu;
    if (base == "wq") { dst = L.wqkv; n = Hq * dh * d * 2; }
    else if (base == "wk") { dst = L.wqkv + Hq * dh * d; n = Hkv * dh * d * 2; }
    else if (base == "wv") { dst = L.wqkv + (Hq + Hkv) * dh * d; n = Hkv * dh * d * 2; }
    else if (base == "wo") { dst = L.wo; n = d * Hq * dh * 2; }
    else if (base == "wr") { dst = L.wr; n = E * d * 2; }
    // gate/up rows are interleaved per group (row 2f gate, 2f + 1 up; group 0 shared):
    // the (expert, f) rows of one kind are every second row from the group's first
    else if (base == "wg") { dst = gu + 2 * F * d; rows = E * F; }
    else if (base == "wu") { dst = gu + 2 * F * d + d; rows = E * F; }
    else if (base == "sg") { dst = gu; rows = F; }
    else if (base == "su") { dst = gu + d; rows = F; }
    else if (base == "wd") { dst = L.wd + d * F; n = E * d * F * 2; }
    else if (base == "sd") { dst = L.wd; n = d * F * 2; }
    else if (base == "ln_in") { dst = L.ln_in; n = d * 4; }
    else if (base == "ln_post") { dst = L.ln_post; n = d * 4; }
    else if (base == "ln_ff") { dst = L.ln_ff; n = d * 4; }
    else return fail(c, DG_ERR_INVALID_ARG, "unknown tensor name");
    if ((base == "sg" || base == "su") && cf.n_shared == 0)
      return fail(c, DG_ERR_INVALID_ARG, "the config has no shared expert");
    if (base == "wg" || base == "wu" || base == "sg" || base == "su" || base == "wd" || base == "sd")
      requant_layer = &L;
    if (rows) { row_bytes = d * 2; pitch = 2 * d * 2; n = rows * row_bytes; }
  }
  if (bytes != n) return fail(c, DG_ERR_INVALID_ARG, "byte count does not match the tensor");
  if (rows)
    DG_CUDA(c, cudaMemcpy2DAsync(dst, pitch, src, row_bytes, row_bytes, rows, cudaMemcpyDefault,
                                 c->stream));
  else
    DG_CUDA(c, cudaMemcpyAsync(dst, src, n, cudaMemcpyDefault, c->stream));
  if (requant_layer) {   // an expert tensor changed: its FP8 codes follow
    const int rc = quantize_layer(c, *requant_layer);
    if (rc != DG_OK) return rc;
  }
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  return DG_OK;
}

int dg_debug_tensor(dg_ctx* c, const char* name, void* dst, size_t bytes, size_t* bytes_needed) {
  if (!c || !name) return DG_ERR_INVALID_ARG;
  const dg_config& cf = c->cfg;
  const size_t T = c->last_T, d = cf.d_model, E = cf.n_experts, k = cf.top_k;
  const size_t dh = cf.head_dim, Hq = cf.n_q_heads, Hkv = cf.n_kv_heads;
  const void* src = nullptr;
  size_t n = 0;
  const std::string s(name);
  if (s == "x" || s == "hn") { src = c->x; n = T * d * 2; }
  else if (s == "q") { src = c->q; n = T * Hq * dh * 2; }
  else if (s == "kc") { src = c->kc; n = T * Hkv * dh * 2; }
  else if (s == "vc") { src = c->vc; n = T * Hkv * dh * 2; }
  else if (s == "attn_o") { src = c->attn_o; n = T * Hq * dh * 2; }
  else if (s == "h") { src = c->h; n = T * d * 4; }
  else if (s == "x2") { src = c->xperm; n = T * d * 2; }
  else if (s == "router_logits") { src = c->router_logits; n = T * E * 4; }
  else if (s == "idx") { src = c->idx; n = T * k * 4; }
  else if (s == "w") { src = c->w; n = T * k * 4; }
  else if (s == "offsets") { src = c->offsets_r; n = (E + 1) * 4; }
  else if (s == "perm") { src = c->perm; n = T * k * 4; }
  else if (s == "tok") { src = c->tok; n = T * 4; }
  else if (s == "conf") { src = c->conf; n = T * 4; }
  else if (s == "head_max") { src = c->head_max; n = T * 4; }
  else if (s == "entropy") { src = c->eb_H; n = T * 4; }
  else if (s == "eb_drawn") { src = c->eb_drawn; n = T * 4; }
  else if (s == "embed") { src = c->embed; n = (size_t)cf.vocab * d * 2; }
  else if (s == "expert_active") { src = c->expert_active; n = (size_t)cf.n_layers * 4; }
  else {
    // weights of one layer: "<name>:<layer>"
    const size_t colon = s.find(':');
    if (colon == std::string::npos) return fail(c, DG_ERR_INVALID_ARG, "unknown tensor name");
    const std::string base = s.substr(0, colon);
    const int l = std::atoi(s.c_str() + colon + 1);
    if (l < 0 || l >= cf.n_layers) return fail(c, DG_ERR_INVALID_ARG, "layer out of range");
    const Layer& L = c->layers[l];
    const size_t F = cf.d_ff;
    if (base == "wqkv") { src = L.wqkv; n = (size_t)c->NQKV * d * 2; }
    else if (base == "wo") { src = L.wo; n = d * Hq * dh * 2; }
    else if (base == "wr") { src = L.wr; n = E * d * 2; }
    else if (base == "wgu") { src = L.wgu; n = (size_t)c->G * 2 * F * d * 2; }
    else if (base == "wd") { src = L.wd; n = (size_t)c->G * d * F * 2; }
    else if (base == "wgu8" && L.wgu8) { src = L.wgu8; n = (size_t)c->G * 2 * F * d; }
    else if (base == "sgu" && L.sgu) { src = L.sgu; n = (size_t)c->G * 2 * F * 4; }
    else if (base == "wd8" && L.wd8) { src = L.wd8; n = (size_t)c->G * d * F; }
    else if (base == "sd8" && L.sd8) { src = L.sd8; n = (size_t)c->G * d * 4; }
    else return fail(c, DG_ERR_INVALID_ARG, "unknown tensor name");
  }
  if (bytes_needed) *bytes_needed = n;
  if (!dst) return DG_OK;
  if (bytes < n) return fail(c, DG_ERR_INVALID_ARG, "destination too small");
  DG_CUDA(c, cudaMemcpyAsync(dst, src, n, cudaMemcpyDefault, c->stream));
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  return DG_OK;
}

int dg_profile_enable(dg_ctx* c, int on) {
  if (!c) return DG_ERR_INVALID_ARG;
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  c->prof.clear();
  c->prof_on = on != 0;
  if (on) DG_CUDA(c, cudaMemset(c->expert_active, 0, sizeof(int) * c->cfg.n_layers));
  return DG_OK;
}

int dg_profile_read(dg_ctx* c, const char* kernel, double* total_ms, int* launches) {
  if (!c || !kernel || !total_ms || !launches) return DG_ERR_INVALID_ARG;
  int kind = -1;
  for (int i = 0; i < K_NUM_KINDS; ++i)
    if (std::string(kernel) == kKindNames[i]) kind = i;
  if (kind < 0) return fail(c, DG_ERR_INVALID_ARG, "unknown kernel name");
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  double t = 0.0;
  int n = 0;
  for (const auto& r : c->prof) {
    if (r.kind != kind) continue;
    float ms = 0.f;
    DG_CUDA(c, cudaEventElapsedTime(&ms, r.a, r.b));
    t += ms;
    ++n;
  }
  *total_ms = t;
  *launches = n;
  return DG_OK;
}

const char* dg_kernel_name(int i) { return (i >= 0 && i < K_NUM_KINDS) ? kKindNames[i] : nullptr; }

int dg_sync(dg_ctx* c) {
  if (!c) return DG_ERR_INVALID_ARG;
  DG_CUDA(c, cudaStreamSynchronize(c->stream));
  return read_device_error(c);
}

const char* dg_last_error(const dg_ctx* c) {
  return c ? c->err.c_str() : g_create_error.c_str();
}

size_t dg_device_bytes(const dg_ctx* c) { return c ? c->bytes : 0; }

int dg_last_launch_count(const dg_ctx* c) { return c ? c->launches : 0; }

void dg_destroy(dg_ctx* c) {
  if (!c) return;
  cudaStreamSynchronize(c->stream);
  for (cudaEvent_t e : c->ev_pool) cudaEventDestroy(e);
  drop_graphs(c);
  free_all(c);
  delete c;
}

}  // extern "C"
