// Router: top-k expert selection per canvas row and the stable grouping of
// the (row, slot) assignments by expert, in one kernel.
//
// One warp per row: the row's logits (split-K partials of the router GEMM,
// summed in split order, plus the optional bias) are held 8 per lane; k rounds
// of a warp-wide (value desc, index asc) argmax pick the experts; the weights
// are the softmax over the chosen logits; each choice sets the row's bit in an
// expert-membership bitmap.  The last block to finish (a device counter) then
// runs a counting sort over the bitmap: per-expert counts, offsets, and each
// assignment's position = offset + rows with the same expert before it.
// Positions therefore follow row order inside an expert, with no float atomics.
#include <algorithm>

#include "gemm_shared.cuh"

namespace dg {

namespace {
constexpr int kRouterThreads = 256;
constexpr int kRowsPerBlock = kRouterThreads / 32;
constexpr int kRouterMaxSmem = 200 * 1024;   // the grouping's shared-memory limit
}  // namespace

// Top-k of one row whose logits (bias not yet added) lane holds as v[i] for the
// experts e = 128 * (i >> 2) + 4 * lane + (i & 3); writes logits_out, idx, w and
// the row's membership bits.  sel_v / sel_i: 32-entry scratch of this warp.
__device__ __forceinline__ void router_row_topk(const RouterArgs& a, int t, float (&v)[8],
                                                float* sel_v, int* sel_i, int lane) {
  const int E = a.E, k = a.k;
  const int W = (a.T + 31) / 32;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = 128 * (i >> 2) + 4 * lane + (i & 3);
    float x = -INFINITY;
    if (e < E) {
      x = v[i] + (a.bias ? a.bias[e] : 0.f);
      if (a.logits_out) a.logits_out[(size_t)t * E + e] = x;
      if (x != x) x = -INFINITY;
    }
    v[i] = x;
  }
  unsigned taken = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = 128 * (i >> 2) + 4 * lane + (i & 3);
      if (e < E && !(taken & (1u << i)) && (v[i] > bv || (v[i] == bv && e < bi))) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (bi >= 0 && bi < E && ((bi & 127) >> 2) == lane)
      taken |= 1u << (4 * (bi >> 7) + (bi & 3));
    if (lane == 0) {
      sel_v[j] = bv;
      sel_i[j] = bi;
    }
  }
  __syncwarp();
  if (lane < k) {
    const float mx = sel_v[0];
    float den = 0.f;
    for (int j = 0; j < k; ++j) den += __expf(sel_v[j] - mx);
    int e = sel_i[lane];
    if (e < 0 || e >= E) { raise_error(a.err, kErrFault); e = 0; }
    a.idx[(size_t)t * k + lane] = e;
    a.w[(size_t)t * k + lane] = __expf(sel_v[lane] - mx) / den;
    atomicOr(a.bitmap + (size_t)e * W + (t >> 5), 1u << (t & 31));
  }
}

// Elects the block that finished last (a device counter); every thread gets the answer.
__device__ __forceinline__ bool router_last_block(const RouterArgs& a) {
  __shared__ int s_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(a.counter, 1) == (int)(gridDim.x * gridDim.y * gridDim.z) - 1;
  }
  __syncthreads();
  const bool last = s_last;
  if (last) __threadfence();
  return last;
}

// The grouping, run by every thread of the last block: a counting sort over the
// membership bitmap (per-expert counts, offsets, each assignment's position =
// offset + rows of the same expert before it), the chunk tables and order of the
// expert GEMMs, then the counters of the next layer reset.  sm_dyn: at least
// router_smem_bytes(T, E) bytes of shared memory.
__device__ void router_group(const RouterArgs& a, int* sm_dyn) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = a.T, E = a.E, k = a.k;
  const int W = (T + 31) / 32;
  int* prefix = sm_dyn;          // [E * W]
  int* count = sm_dyn + E * W;   // [E]
  int* off = count + E;          // [E + 1]
  uint32_t* words = reinterpret_cast<uint32_t*>(off + E + 1);  // [E * W]
  int* cpre = reinterpret_cast<int*>(words + E * W);   // [E + 2] chunk prefix of the groups
  int* fbase = cpre + E + 2;                           // [E + 1] first order slot of a group's full chunks
  int* prow = fbase + E + 1;                           // [E + 1] rows of a group's partial chunk
  __shared__ int s_total_full;
  for (int i = threadIdx.x; i < E * W; i += blockDim.x) {
    const uint32_t wv = __ldcg(a.bitmap + i);
    words[i] = wv;
    prefix[i] = __popc(wv);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < W; ++w) {
      const int c = prefix[e * W + w];
      prefix[e * W + w] = run;
      run += c;
    }
    count[e] = run;
  }
  __syncthreads();
  if (warp == 0) {
    // offsets and chunk counts: an exclusive scan over the experts, lane l
    // taking the `per` consecutive experts from l * per (integer arithmetic,
    // so the result equals the sequential scan)
    const int per = (E + 31) / 32;
    const int base_chunks = a.n_shared ? (T + a.n_tile - 1) / a.n_tile : 0;
    const int base_full = a.n_shared ? T / a.n_tile : 0;
    int c_cnt = 0, c_chk = 0, c_act = 0, c_full = 0;
    for (int q = 0; q < per; ++q) {
      const int e = lane * per + q;
      if (e < E) {
        c_cnt += count[e];
        c_chk += (count[e] + a.n_tile - 1) / a.n_tile;
        c_act += count[e] > 0;
        c_full += count[e] / a.n_tile;
      }
    }
    int s_cnt = c_cnt, s_chk = c_chk, s_full = c_full;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int vc = __shfl_up_sync(0xffffffffu, s_cnt, o);
      const int vk = __shfl_up_sync(0xffffffffu, s_chk, o);
      const int vf = __shfl_up_sync(0xffffffffu, s_full, o);
      if (lane >= o) { s_cnt += vc; s_chk += vk; s_full += vf; }
    }
    int run = s_cnt - c_cnt;
    int crun = base_chunks + s_chk - c_chk;
    int frun = base_full + s_full - c_full;
    for (int q = 0; q < per; ++q) {
      const int e = lane * per + q;
      if (e < E) {
        off[e] = run;
        if (a.offsets_r) a.offsets_r[e] = run;
        if (a.offsets_g) a.offsets_g[e + 1] = T + run;
        run += count[e];
        cpre[e + 1] = crun;
        fbase[e + 1] = frun;
        crun += (count[e] + a.n_tile - 1) / a.n_tile;
        frun += count[e] / a.n_tile;
        if (a.chunk_prefix) a.chunk_prefix[e + 2] = crun;
      }
    }
    if (lane == 31) {
      cpre[E + 1] = crun;
      s_total_full = frun;
    }
    const int total = __shfl_sync(0xffffffffu, s_cnt, 31);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c_act += __shfl_xor_sync(0xffffffffu, c_act, o);
    if (lane == 0) {
      cpre[0] = 0;
      fbase[0] = 0;
      if (a.offsets_g) a.offsets_g[0] = 0;
      if (a.chunk_prefix) { a.chunk_prefix[0] = 0; a.chunk_prefix[1] = base_chunks; }
      off[E] = total;
      if (a.offsets_r) a.offsets_r[E] = total;
      if (a.offsets_g) a.offsets_g[E + 1] = T + total;
      if (a.active_out) atomicAdd(a.active_out, c_act);
      if (total != T * k) raise_error(a.err, kErrFault);
    }
  }
  __syncthreads();
  if (a.chunk_order) {
    // The grouped GEMMs deal their tiles longest chunk first: the full chunks in
    // chunk order, then each group's partial chunk by decreasing rows (ties
    // toward the lower chunk).  Group 0 is the shared expert (T rows), group
    // e + 1 expert e.
    const int G = E + 1;
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
      const int cnt = g == 0 ? (a.n_shared ? T : 0) : count[g - 1];
      prow[g] = cnt % a.n_tile;
      const int nfull = cnt / a.n_tile;
      for (int j = 0; j < nfull; ++j) a.chunk_order[fbase[g] + j] = cpre[g] + j;
    }
    __syncthreads();
    const int total_full = s_total_full;
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
      const int r = prow[g];
      if (r == 0) continue;
      int rank = 0;
      for (int g2 = 0; g2 < G; ++g2) rank += prow[g2] > r || (prow[g2] == r && g2 < g);
      a.chunk_order[total_full + rank] = cpre[g + 1] - 1;
    }
  }
  for (int i0 = 0; i0 < T * k; i0 += 8 * (int)blockDim.x) {  // 8 index loads in flight per thread
    int ev[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * (int)blockDim.x + threadIdx.x;
      ev[u] = (i < T * k) ? __ldcg(a.idx + i) : -1;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * (int)blockDim.x + threadIdx.x;
      const int e = ev[u];
      if (i >= T * k || e < 0 || e >= E) continue;
      const int tt = i / k;
      const uint32_t word = words[e * W + (tt >> 5)];
      const int pos = off[e] + prefix[e * W + (tt >> 5)] + __popc(word & ((1u << (tt & 31)) - 1u));
      a.perm[pos] = i;
      a.inv[i] = pos;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E * W; i += blockDim.x) a.bitmap[i] = 0u;
  // the expert GEMMs' per-chunk ready counters start this layer at zero
  if (a.chunk_ready)
    for (int i = threadIdx.x; i < a.n_chunk_ready; i += blockDim.x) a.chunk_ready[i] = 0;
  // and so do their tile counters
  if (a.tile_counters && threadIdx.x < a.n_tile_counters) a.tile_counters[threadIdx.x] = 0;
  if (threadIdx.x == 0) *a.counter = 0;
}

__global__ void __launch_bounds__(kRouterThreads) router_kernel(RouterArgs a) {
  extern __shared__ int sm_dyn[];
  __shared__ float s_sel_v[kRowsPerBlock][32];
  __shared__ int s_sel_i[kRowsPerBlock][32];
  griddep_wait();
  griddep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = a.T, E = a.E;
  const int t = blockIdx.x * kRowsPerBlock + warp;
  if (t < T) {
    // lane holds experts e = 128 * hh + 4 * lane + q
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
    // the two expert halves in turn (E <= 256), 16 splits' loads in flight at once;
    // each logit sums its splits in split order
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int e0 = 128 * hh + 4 * lane;
      if (128 * hh >= E) break;
      for (int s0 = 0; s0 < a.splits; s0 += 16) {
        float4 buf[16];
#pragma unroll
        for (int ss = 0; ss < 16; ++ss)
          if (s0 + ss < a.splits && e0 < E)
            buf[ss] = __ldg(reinterpret_cast<const float4*>(
                a.logits_in + ((size_t)(s0 + ss) * T + t) * E + e0));
#pragma unroll
        for (int ss = 0; ss < 16; ++ss)
          if (s0 + ss < a.splits && e0 < E) {
            v[4 * hh + 0] += buf[ss].x; v[4 * hh + 1] += buf[ss].y;
            v[4 * hh + 2] += buf[ss].z; v[4 * hh + 3] += buf[ss].w;
          }
      }
    }
    router_row_topk(a, t, v, s_sel_v[warp], s_sel_i[warp], lane);
  }
  if (!router_last_block(a)) return;
  router_group(a, sm_dyn);
}

// ---------------------------------------------------------------- logits, top-k and grouping

// The router with its logits GEMM in one kernel.  A cluster of S CTAs takes one
// tile of n_tile token rows: CTA r computes the partial logits over its share of
// the hidden dimension on the tensor cores (tcgen05, M = 128 experts x N = the
// tile's rows, accumulator in TMEM), stores them in its shared memory as
// [row][128 experts] fp32, and after a cluster barrier sums, for its own
// n_tile / S rows, the S partials in rank order with distributed shared-memory
// loads.  Then each row's top-k as in the router kernel, a second cluster barrier
// (no CTA leaves while another reads its shared memory), and the grid's last CTA
// groups.  Experts beyond E read zero weight rows and are skipped.  E <= 128.
namespace {

// warps 0..5 run the GEMM (producer, MMA, four TMEM readers); all 16 warps then
// reduce and rank rows, two or so per warp
constexpr int kFusedThreads = 512;
constexpr int kFusedStages = 4;

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// A load from another CTA's shared memory; ordered after the cluster barrier that
// precedes it (a volatile asm with a memory clobber), free to overlap its peers.
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
      : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
      : "r"(addr));
  return v;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

}  // namespace

__global__ void __launch_bounds__(kFusedThreads, 1)
router_fused_kernel(const __grid_constant__ CUtensorMap mapW, const __grid_constant__ CUtensorMap mapX,
                    const RouterFusedArgs f) {
  const RouterArgs& a = f.r;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ float s_sel_v[kFusedThreads / 32][32];
  __shared__ int s_sel_i[kFusedThreads / 32][32];
  const uint32_t stage_bytes = (uint32_t)kATileBytes + (uint32_t)f.n_tile * 128u;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)f.ring_bytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kFusedStages + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_u32(bars);
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (kFusedStages + s); };
  const uint32_t tfull_bar = bar_base + 8u * (2 * kFusedStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank(), S = cluster_size();
  const int row0 = (int)(blockIdx.x / S) * f.n_tile;            // the cluster's token tile
  const int rows = min(f.n_tile, a.T - row0);
  const int n_mma = (rows + 15) & ~15;
  const int kb0 = (int)(rank * (uint32_t)f.n_kb / S), kb1 = (int)((rank + 1) * (uint32_t)f.n_kb / S);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kFusedStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tfull_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mapW);
    tma_prefetch_desc(&mapX);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();
  griddep_launch();

  bool ok = true;
  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.err)) break;
        const uint32_t sA = smem_base + (uint32_t)stage * stage_bytes;
        mbar_arrive_expect_tx(full_bar(stage), stage_bytes);
        tma_load_2d(sA, &mapW, full_bar(stage), kb * kBK, 0);
        tma_load_2d(sA + kATileBytes, &mapX, full_bar(stage), kb * kBK, row0);
        if (++stage == kFusedStages) { stage = 0; phase ^= 1u; }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16_f32(n_mma);
      int stage = 0;
      uint32_t phase = 0;
      bool mok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(full_bar(stage), phase, abort_flag, a.err)) { mok = false; break; }
        tc_fence_after();
        const uint32_t sA = smem_base + (uint32_t)stage * stage_bytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          umma_bf16(tmem_base, sdesc_kmajor_sw128(sA + kk * 32),
                    sdesc_kmajor_sw128(sA + kATileBytes + kk * 32), idesc,
                    (kb > kb0 || kk > 0) ? 1u : 0u);
        umma_commit(empty_bar(stage));
        if (++stage == kFusedStages) { stage = 0; phase ^= 1u; }
      }
      if (mok) umma_commit(tfull_bar);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ---------------------------------------------- accumulator -> shared memory
    // lane = expert (its quadrant of TMEM lanes), column = token row; stored as
    // part[row][128] over the operand ring, idle once every MMA has completed
    const int q = warp & 3;
    ok = __all_sync(0xffffffffu, mbar_wait(tfull_bar, 0, abort_flag, a.err));
    if (ok) {
      tc_fence_after();
      float* part = reinterpret_cast<float*>(smem);
      uint32_t v[32];
      for (int c0 = 0; c0 < n_mma; c0 += 32) {
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) part[(c0 + j) * 128 + q * 32 + lane] = __uint_as_float(v[j]);
      }
    }
  }
  // every CTA's partials are in its shared memory
  tc_fence_before();
  cluster_sync_all();
  // this CTA's rows of the tile: the S partials summed in rank order, then top-k
  {
    const int r0 = (int)(rank * (uint32_t)f.n_tile / S), r1 = (int)((rank + 1) * (uint32_t)f.n_tile / S);
    const uint32_t part_base = smem_base;
    for (int rr = r0 + warp; rr < r1 && rr < rows; rr += kFusedThreads / 32) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
      const uint32_t off = part_base + (uint32_t)(rr * 128 + 4 * lane) * 4u;
      float4 p[8];
#pragma unroll
      for (int src = 0; src < 8; ++src)      // every rank's loads in flight at once
        if (src < (int)S) p[src] = ld_cluster_f4(map_to_rank(off, (uint32_t)src));
#pragma unroll
      for (int src = 0; src < 8; ++src)      // summed in rank order
        if (src < (int)S) { v[0] += p[src].x; v[1] += p[src].y; v[2] += p[src].z; v[3] += p[src].w; }
      router_row_topk(a, row0 + rr, v, s_sel_v[warp], s_sel_i[warp], lane);
    }
  }
  // no CTA reuses or leaves its shared memory while another may still read it
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
  if (!router_last_block(a)) return;
  router_group(a, reinterpret_cast<int*>(smem));
}

size_t router_fused_smem_bytes(const RouterFusedArgs& f) {
  // alignment slack, the operand ring (also holding the partials and the grouping's
  // tables in turn), barriers
  return 1024 + (size_t)f.ring_bytes + 256;
}

cudaError_t launch_router_fused(const CUtensorMap& mapW, const CUtensorMap& mapX,
                                RouterFusedArgs f, cudaStream_t s) {
  const RouterArgs& a = f.r;
  if (a.E > 128 || f.n_kb < 1 || f.n_tile < 16 || f.n_tile > 256 || f.n_tile % 16 != 0)
    return cudaErrorInvalidValue;
  const int S = f.n_kb < 8 ? f.n_kb : 8;
  const size_t ring = (size_t)kFusedStages * ((size_t)kATileBytes + (size_t)f.n_tile * 128);
  const size_t need = std::max({ring, (size_t)f.n_tile * 512, router_smem_bytes(a.T, a.E)});
  f.ring_bytes = (int)((need + 1023) / 1024 * 1024);
  const size_t smem = router_fused_smem_bytes(f);
  // the dynamic limit leaves room for the kernel's static shared memory
  if (smem > (size_t)kRouterMaxSmem) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(router_fused_kernel),
                                    kRouterMaxSmem);
  if (e != cudaSuccess) return e;
  const int tiles = (a.T + f.n_tile - 1) / f.n_tile;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles * S);
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, router_fused_kernel, mapW, mapX, f);
}

int router_max_smem_bytes() { return kRouterMaxSmem; }

size_t router_smem_bytes(int T, int E) {
  const int W = (T + 31) / 32;
  return (size_t)(2 * E * W + E + E + 1 + 3 * E + 4) * sizeof(int);
}

cudaError_t launch_router(const RouterArgs& a, cudaStream_t s) {
  const size_t smem = router_smem_bytes(a.T, a.E);
  if (smem > (size_t)kRouterMaxSmem) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(router_kernel), kRouterMaxSmem);
  if (e != cudaSuccess) return e;
  return launch_k(router_kernel, dim3((a.T + kRowsPerBlock - 1) / kRowsPerBlock),
                  dim3(kRouterThreads), smem, s, a);
}

}  // namespace dg
