// Internal kernel interfaces of libdg (not part of the C ABI).
#pragma once

#include "dg_common.cuh"

namespace dg {

// Raises the dynamic shared-memory limit of `func` to `bytes` on the current
// device.  The attribute belongs to the device, so this is done once per
// (kernel, device) pair; the table is guarded by a mutex, so host threads
// driving different devices may launch at the same time.
cudaError_t ensure_smem_limit(const void* func, int bytes);

enum GemmMode { GEMM_DENSE = 0, GEMM_GATEUP = 1, GEMM_DOWN = 2, GEMM_HEAD = 3 };

struct GemmArgs {
  int mode;
  int M, N, K, n_kb;      // A rows, B rows, reduction length, K / 64
  int n_tile;             // B rows per tile (DENSE / grouped)
  int k_splits;           // DENSE split-K
  int dense_pair;         // DENSE: tiles of two 128-row slabs (m_slabs counts pairs)
  int m_slabs;            // 128-row slabs of A per group (DENSE / grouped)
  int n_groups;           // grouped: number of groups
  const int* offsets;     // grouped: [n_groups + 1] first B row of each group
  const int* chunk_prefix;// grouped: [n_groups + 1] prefix of ceil(rows_g / n_tile)
  int F;                  // GATEUP output width
  int T, vocab, mask_id;  // HEAD
  int n_vblocks, n_tblocks;
  float* out_f32;
  bf16* out_bf16;
  float* head_m;
  float* head_s;
  int* head_a;
  const float* inv_temp;  // HEAD: NULL, or the inverse temperature (device) for the
  float* head_q;          //   entropy variant, which also writes sum z e^z to head_q
  int* err;
  // shared-memory and TMEM plan (gemm_plan_smem): stages = k-blocks in flight at
  // most, stage_bytes = the largest k-block, ring_bytes = the operand ring
  int stages, a_bytes, b_bytes, stage_bytes, b_box_rows;
  int ring_bytes;
  int n_bufs;
  // Gate/up -> down hand-over without a whole-grid wait: GATEUP adds 1 to
  // chunk_ready[c] per epilogue warp once its H rows of chunk c are written;
  // DOWN (which then skips the grid dependency wait) loads a chunk's H rows
  // once chunk_ready[c] reaches ready_target.  NULL: not used.
  int* chunk_ready;
  int ready_target;
  // Grouped modes: tiles dealt longest chunk first from chunk_order (the router's
  // order, max_chunks entries at most), taken one at a time from *tile_counter
  // (zeroed by the router) when it is not NULL.  pair: a tile covers 256 weight
  // rows (two accumulators; DOWN only).
  const int* chunk_order;
  int* tile_counter;
  int max_chunks;
  int pair;
  const float* w_scale;   // FP8-weight GEMMs: [n_groups][M] fp32 scale of each weight row
  int sa, sb;             // FP8-weight GEMMs: bf16 A and B ring stages (gemm_fp8_plan_smem)
  int tab_bytes;          // group tables in shared memory (grouped modes)
  int epi_bytes;          // fp32 output staging in shared memory (DENSE, DOWN)
};

bool make_tmap_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                  uint32_t box_outer);
bool make_tmap_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid,
                  uint64_t outer, uint32_t box_mid);
// bf16 [outer][inner] map with [32 rows][16] boxes (the gate/up H stores).
bool make_tmap_h_store(CUtensorMap* map, void* base, uint64_t inner, uint64_t outer);
// fp32 [outer][inner] map with 32 x 32 boxes in the 128-byte swizzle (the
// attention's partial-output stores).
bool make_tmap_f32_sw128(CUtensorMap* map, float* base, uint64_t inner, uint64_t outer);
// fp32 [outer][mid][inner] output map for the DENSE / DOWN tensor stores.
bool make_tmap_out_f32(CUtensorMap* map, float* base, uint64_t inner, uint64_t mid,
                       uint64_t outer);
void gemm_plan_smem(GemmArgs& a);
// Two-SM (cta_group::2) dense projection: clusters of two CTAs, each holding one
// 128-row weight slab and half of the tile's activation rows (mapB_half: boxes
// of b_box_rows = n_tile / 2 rows).  DENSE only, m_slabs even.
void gemm_pair_plan_smem(GemmArgs& a);
int gemm_pair_max_clusters();   // co-resident two-CTA clusters of the pair GEMM (0: none)
cudaError_t gemm_pair_launch(const CUtensorMap& mapA, const CUtensorMap& mapB_half,
                             const CUtensorMap& mapC, const GemmArgs& a, int clusters,
                             cudaStream_t stream);
size_t gemm_smem_bytes(const GemmArgs& a);
// mapC: the output map (DENSE: fp32 [k_splits][N][M]; DOWN: fp32 [1][rows][M];
// GATEUP: bf16 H [rows][F]); any valid map for HEAD, which does not use it.
cudaError_t gemm_tc_launch(const CUtensorMap& mapA, const CUtensorMap& mapB,
                           const CUtensorMap& mapC, const GemmArgs& a, int grid,
                           cudaStream_t stream);

// Expert GEMMs with FP8 E4M3 weights (gemm_fp8.cu): GATEUP or DOWN (pair only in
// DOWN), dynamic tiles (tile_counter and w_scale required).  mapW: the codes
// [n_groups][M][K] (uint8, boxes 64 codes x 128 rows, make_tmap_3d_u8).
void gemm_fp8_plan_smem(GemmArgs& a);
cudaError_t gemm_fp8_launch(const CUtensorMap& mapW, const CUtensorMap& mapB,
                            const CUtensorMap& mapC, const GemmArgs& a, int grid,
                            cudaStream_t stream);
bool make_tmap_3d_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid,
                     uint64_t outer);
// bf16 rows [rows][K] -> E4M3 codes [rows][K] + fp32 scales [rows] (one per row).
cudaError_t launch_quantize_rows(const bf16* src, uint8_t* dst, float* scale, long long rows,
                                 int K, cudaStream_t s);

// ---------------------------------------------------------------- weight init
// Physical layouts of the generated tensors (see init kernels).
enum InitLayout {
  INIT_PLAIN = 0,   // physical == logical [rows][cols] of tensor tid
  INIT_QKV = 1,     // rows [0,nq) tid_q, [nq,nq+nkv) tid_k, rest tid_v; cols d
  INIT_GATEUP = 2,  // [E+1][2F][d]: group 0 shared expert, group g>0 expert g-1;
                    // row 2f = gate row f, row 2f+1 = up row f
  INIT_DOWN = 3     // [E+1][d][F]: group 0 shared expert, group g>0 expert g-1
};

struct InitArgs {
  int layout;
  bf16* dst;
  long long n_elems;     // physical elements
  unsigned long long key0, key1, key2, key3;  // stream keys (meaning per layout)
  int rows_a, rows_b;    // QKV: nq, nkv
  int cols;              // innermost width (d or F)
  int F, d, E;           // grouped layouts
  float scale;           // float32(std * sqrt(3) / 65536)
};

unsigned long long stream_key_host(unsigned long long seed, unsigned long long tid);
cudaError_t launch_init(const InitArgs& a, cudaStream_t s);
cudaError_t launch_fill_f32(float* p, long long n, float v, cudaStream_t s);
cudaError_t launch_set_int(int* p, int v, cudaStream_t s);
// kc / vc [B][Hkv][n][dh] -> cache [B][Hkv][C][dh] at positions P0 .. P0 + n - 1.
cudaError_t launch_kv_append(const bf16* kc, const bf16* vc, bf16* ck, bf16* cv, int B, int Hkv,
                             int n, int dh, int C, int P0, cudaStream_t s);

// ---------------------------------------------------------------- elementwise / norm
// h[t] = float(E[canvas[t]]) (or float(x_in[t]) when x_in != NULL);
// x[t] = bf16(rmsnorm(h[t]) * w)
cudaError_t launch_embed_norm(const int32_t* canvas, const bf16* embed, const bf16* x_in,
                              int vocab, int T, int d, const float* w, float eps, float* h,
                              bf16* x, int* err, cudaStream_t s);

// cos/sin table [Tc][dh/2] for positions P + i, in double precision.
cudaError_t launch_rope_table(float* cos_t, float* sin_t, int Tc, int half, int P, double theta,
                              cudaStream_t s);

// Sum QKV split-K partials, rotate q and k (first n_rot pairs), scatter to
// q [B][Hq][Tc][dh], kc/vc [B][Hkv][Tc][dh] (bf16).
cudaError_t launch_qkv_rope(const float* part, int splits, int T, int Tc, int Hq, int Hkv, int dh,
                            int n_rot, const float* cos_t, const float* sin_t, bf16* q, bf16* kc,
                            bf16* vc, cudaStream_t s);

// The split-KV attention partials, as the merge reads them: per key-range
// chunk c and query row R = (b * Hq + h) * Tc + i, the un-normalised O
// (part_o[c][R][dh]) and (m, l) with m in log2 units (part_ml[c][R][2]).
struct AttnMergeArgs {
  int B, Hq, Tc, dh;
  int n_chunks;
  const float* part_o;   // [n_chunks][B*Hq*Tc][dh]
  const float* part_ml;  // [n_chunks][B*Hq*Tc][2]
};

// tcgen05 attention (attention_tc.cu): writes the split-KV partials part_o /
// part_ml in the AttnMergeArgs layout above; launch_attn_merge (attn_merge.cu)
// combines them.
struct AttnTcArgs {
  int B, Hq, Hkv, Tc, P, dh;
  int n_vis;
  // Rows per (sequence, kv head) in the prompt K/V maps: P for a caller's cache,
  // the capacity for the library's own.
  int kv_stride;
  // Causal attention (the encoder): new token i (position P + i) sees the cached
  // and new positions <= P + i, and with window > 0 only those >= P + i - window + 1.
  // n_vis then covers the widest row's cached range.  0: the decoder's joint softmax.
  int causal, window;
  int n_chunks;          // key-block ranges per (canvas, kv head, query tile)
  float* part_o;         // [n_chunks][B*Hq*Tc][dh]
  float* part_ml;        // [n_chunks][B*Hq*Tc][2]
  float scale_log2;
  int* err;
  // 1: the n_chunks CTAs of a query tile run as one cluster and merge in shared
  // memory into `out` (n_chunks <= 8; part_o / part_ml unused); 0: partials
  int fused;
  bf16* out;             // [T][Hq*dh] bf16 (t = b*Tc + i), as the merge kernel writes
};
struct AttnTcMaps {
  CUtensorMap q;         // [B*Hq*Tc][dh], box 64 x 128 rows
  CUtensorMap kc, vc;    // [B*Hkv*Tc][dh], box 64 x 64 rows
  CUtensorMap kp, vp;    // [B*Hkv*P][dh],  box 64 x 64 rows
  CUtensorMap po;        // part_o as [chunks * rows][dh] fp32, box 32 x 32, 128-byte swizzle
};
int attn_tc_blocks(int n_vis, int Tc);
int attn_tc_qtiles(int Hq, int Hkv, int Tc);
cudaError_t launch_attention_tc(const AttnTcMaps& m, const AttnTcArgs& a, cudaStream_t s);
// Whether the cluster-merged form can run with this head width and range count on
// the current device (at most 8 ranges, and the cluster fits the GPU).
bool attn_tc_fused_ok(int dh, int n_chunks);
// Merge partials -> o [T][Hq*dh] bf16 (t = b*Tc + i)
cudaError_t launch_attn_merge(const AttnMergeArgs& a, bf16* o, cudaStream_t s);

// a = sum of O-projection partials; h1 = h + rmsnorm(a)*w_post (h updated in
// place); x2 = bf16(rmsnorm(h1)*w_ff).
cudaError_t launch_post_attn(const float* part, int splits, int T, int d, const float* w_post,
                             const float* w_ff, float eps, float* h, bf16* x2, cudaStream_t s);

// Router (one kernel): logits = sum of split-K partials (+ bias); top-k per row
// (value desc, index asc); weights = softmax over the chosen logits; then the
// last block groups the assignments by expert.  Routed offsets_r [E+1] and
// perm/inv [T*k] are relative to the routed block; offsets_g / chunk_prefix
// [E+2] describe the grouped-GEMM groups: group 0 = shared expert rows
// [0, T), group e+1 = expert e rows [T + offsets_r[e], T + offsets_r[e+1]).
// The bitmap must be zero on entry and is left zero; counter likewise.
struct RouterArgs {
  const float* logits_in;  // [splits][T][E] fp32
  int splits;
  const float* bias;       // [E] or NULL
  int T, E, k, n_shared, n_tile;
  float* logits_out;       // [T][E] or NULL
  int32_t* idx;            // [T][k]
  float* w;                // [T][k]
  uint32_t* bitmap;        // [E][ceil(T/32)]
  int* counter;            // one int, zero on entry
  int32_t* offsets_r;      // [E+1] or NULL
  int32_t* offsets_g;      // [E+2] or NULL
  int32_t* chunk_prefix;   // [E+2] or NULL
  int32_t* perm;           // [T*k]
  int32_t* inv;            // [T*k]
  int* active_out;         // += experts given rows, or NULL
  int* chunk_ready;        // [n_chunk_ready] set to 0 (the expert GEMMs' counters), or NULL
  int n_chunk_ready;
  int32_t* chunk_order;    // [n_chunk_ready] chunks longest first (the GEMMs' tile order), or NULL
  int* tile_counters;      // [n_tile_counters] set to 0 (the GEMMs' dynamic tile counters), or NULL
  int n_tile_counters;
  int* err;
};
size_t router_smem_bytes(int T, int E);
int router_max_smem_bytes();   // launch_router refuses larger shared-memory plans
cudaError_t launch_router(const RouterArgs& a, cudaStream_t s);
// The router with its logits GEMM (E <= 128): logits = X W^T on the tensor cores,
// split over the hidden dimension across a cluster of min(8, n_kb) CTAs per tile of
// n_tile token rows and summed in rank order through distributed shared memory;
// then top-k and the grouping as launch_router.  mapW: the router weights
// [>=128][d] bf16 (128-row boxes), mapX: the normed rows [T..][d] (n_tile-row boxes).
// logits_in / splits of r are not used.
struct RouterFusedArgs {
  RouterArgs r;
  int n_kb;         // d / 64
  int n_tile;       // token rows per cluster (the B box height), a multiple of 16, <= 256
  int ring_bytes;   // set by the launcher
};
cudaError_t launch_router_fused(const CUtensorMap& mapW, const CUtensorMap& mapX,
                                RouterFusedArgs f, cudaStream_t s);
// xperm[T + p] = xperm[perm[p] / k] for p < k*T (rows [0, T) hold the normed input).
cudaError_t launch_moe_gather(bf16* xperm, const int32_t* perm, int T, int k, int d,
                              cudaStream_t s);
// h = h + sum_j w[t][j] Y[T + inv[t*k+j]] (+ Y[t] shared); then either
// x = bf16(rmsnorm(h)*w_next) (w_next != NULL) or x = bf16(h).
cudaError_t launch_moe_combine(const float* Y, const float* w, const int32_t* inv, int T, int k,
                               int n_shared, int d, float* h, const float* w_next, float eps,
                               bf16* x, cudaStream_t s);

// Vocab head merge over vocab blocks: conf = 1/sum, tok = argmax, max_logit = max.
cudaError_t launch_head_merge(const float* hm, const float* hs, const int* ha, int n_vblocks,
                              int T, float* conf, int32_t* tok, float* max_logit,
                              cudaStream_t s);
// Entropy-bounded pass (eb_sampler.cu).  eb_merge folds the HEAD partials taken at
// inverse temperature *inv_temp into per row: H (entropy, nats), tok (argmax),
// max_logit and sum = sum_v e^((l_v - max) * inv_temp).
struct EbMergeArgs {
  int T, n_vblocks;
  const float* hm;
  const float* hs;
  const float* hq;
  const int* ha;
  const float* inv_temp;
  float* H;
  int32_t* tok;
  float* max_logit;
  float* sum;
};
cudaError_t launch_eb_merge(const EbMergeArgs& a, cudaStream_t s);

// One CTA per canvas: the stop test, then the commit at a stop / the last pass
// (argmax tokens) or by the entropy bound (drawn tokens; drawn_in given: those
// tokens, no draw).  state[b] (optional): bit 0 = prev_in holds the previous
// pass's argmax, bit 1 = the canvas is done (left unchanged).
struct EbCommitArgs {
  int B, Tc, T, mask_id, vocab, d, n_vblocks;
  const float* H;
  const int32_t* argmax;
  const int32_t* drawn_in;   // NULL: draw from the head partials
  const float* u;            // [T] uniforms of the draw
  const bf16* hn;            // [T][d] the states the head read
  const bf16* embed;         // [vocab][d]
  const float* head_m;       // [n_vblocks][T]
  const float* head_s;
  const float* max_logit;    // [T] (eb_merge)
  const float* sum;          // [T]
  const float* inv_temp;
  const int32_t* prev_in;    // [T] previous argmax or NULL
  const int* state;          // [B] or NULL
  int32_t* prev_out;         // [T] or NULL
  int* state_out;            // [B] or NULL
  const int* last_flag;      // device flag "last allowed pass", or NULL: use `last`
  int last;
  double bound, threshold;
  int32_t* canvas;
  uint8_t* committed;        // [T] or NULL
  uint8_t* stopped;          // [B] or NULL
  int32_t* drawn_out;        // [T] or NULL: the drawn token of each committed slot
};
cudaError_t launch_eb_commit(const EbCommitArgs& a, cudaStream_t s);
cudaError_t launch_set_float(float* p, float v, cudaStream_t s);

// Commit (one block per canvas).  steps_left read from *steps_left_dev when
// steps_left < 0.
cudaError_t launch_commit(const float* conf, const int32_t* tok, int32_t* canvas,
                          uint8_t* committed, int B, int Tc, int steps_left,
                          const int* steps_left_dev, int mask_id, cudaStream_t s);

}  // namespace dg
