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
#include "dg_kernels.h"

namespace dg {

namespace {
constexpr int kRouterThreads = 256;
constexpr int kRowsPerBlock = kRouterThreads / 32;
constexpr int kRouterMaxSmem = 200 * 1024;   // the grouping's shared-memory limit
}  // namespace

__global__ void __launch_bounds__(kRouterThreads) router_kernel(RouterArgs a) {
  extern __shared__ int sm_dyn[];
  __shared__ float s_sel_v[kRowsPerBlock][32];
  __shared__ int s_sel_i[kRowsPerBlock][32];
  __shared__ int s_last;
  griddep_wait();
  griddep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = a.T, E = a.E, k = a.k;
  const int W = (T + 31) / 32;
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
        s_sel_v[warp][j] = bv;
        s_sel_i[warp][j] = bi;
      }
    }
    __syncwarp();
    if (lane < k) {
      const float mx = s_sel_v[warp][0];
      float den = 0.f;
      for (int j = 0; j < k; ++j) den += __expf(s_sel_v[warp][j] - mx);
      int e = s_sel_i[warp][lane];
      if (e < 0 || e >= E) { raise_error(a.err, kErrFault); e = 0; }
      a.idx[(size_t)t * k + lane] = e;
      a.w[(size_t)t * k + lane] = __expf(s_sel_v[warp][lane] - mx) / den;
      atomicOr(a.bitmap + (size_t)e * W + (t >> 5), 1u << (t & 31));
    }
  }

  // ------------------------------------------------ the last block sorts
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(a.counter, 1) == (int)gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
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
  for (int i0 = 0; i0 < T * k; i0 += 8 * kRouterThreads) {  // 8 index loads in flight per thread
    int ev[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * kRouterThreads + threadIdx.x;
      ev[u] = (i < T * k) ? __ldcg(a.idx + i) : -1;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * kRouterThreads + threadIdx.x;
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
