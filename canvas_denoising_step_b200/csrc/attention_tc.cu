// Canvas attention on the 5th-generation tensor cores (tcgen05).
//
// One softmax over {the visible prompt keys} U {all canvas keys} for every
// canvas query row, with grouped-query heads.  A CTA takes 128 query rows of
// one (canvas b, kv head g) -- the rows of the group's query heads, stacked --
// and one contiguous range of 64-key blocks.  Prompt-key blocks and canvas-key
// blocks are kept apart so that every block is one TMA box from one source.
//
// Roles (192 threads):
//   warp 0, lane 0   TMA: the Q tile once, then K and V of each key block
//                    into a two-stage ring (K and V share the layout
//                    [dh/64][64 keys][128 B], 128-byte swizzle);
//   warp 1           TMEM allocation; lane 0 issues the MMAs:
//                    S_j = Q K_j^T into one of two S buffers (M=128, N=64),
//                    then O += P_{j-1} V_{j-1} (M=128, N=dh, V as an MN-major
//                    operand) once the softmax has written P_{j-1};
//   warps 2..5       softmax, one query row per thread: read S_j from TMEM,
//                    mask and scale (log2 units), keep a reference max m and
//                    the running sum l; when a block's max exceeds m by more
//                    than 8 (a factor 256) O is rescaled in TMEM, otherwise the
//                    stale m is kept (P <= 256 stays exact enough in bf16);
//                    write P_j as bf16 into shared memory in the K-major
//                    128-byte-swizzle layout the MMA reads.
// The CTA's result is the un-normalised partial (O, m, l) of its key range.
// With the in-cluster merge (the key ranges of one query tile launched as one
// thread-block cluster of at most 8 CTAs) every CTA stages its partial in its own
// shared memory, and after a cluster barrier CTA c combines rows
// [128c/C, 128(c+1)/C) of all C partials by log-sum-exp, reading its peers'
// shared memory (distributed shared memory), and writes the bf16 output the
// output projection reads; a second cluster barrier keeps every CTA resident
// until its peers have read it.  Otherwise the partials go to global memory and
// the merge kernel (attn_merge.cu) combines them, with the same arithmetic in the
// same order, so the two routes give the same bits.
#include <climits>
#include <map>
#include <mutex>
#include <tuple>

#include "dg_kernels.h"

namespace dg {

namespace {

constexpr int kThreads = 192;
constexpr int kBN = 64;          // keys per block
constexpr int kRows = 128;       // query rows per CTA
constexpr int kStages = 2;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kMaxClusterChunks = 8;       // key ranges merged inside one cluster
constexpr int kWStride = kMaxClusterChunks + 1;   // a merged row's weights, then 1 / L

__device__ __forceinline__ uint32_t attn_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// the address of the same shared-memory location in the cluster's CTA `rank`
__device__ __forceinline__ uint32_t attn_mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ float4 attn_ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ float2 attn_ld_cluster_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
  return v;
}

// every thread of every CTA of the cluster; the writes before it are seen after it
__device__ __forceinline__ void attn_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

template <int DH>
struct AttnSmem {
  static constexpr int kQ = kRows * DH * 2;         // Q tile
  static constexpr int kKV = kBN * DH * 2;          // one K (or V) block
  static constexpr int kP = kRows * kBN * 2;        // P tile
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQ;                  // [stage] K
  static constexpr int kVOff = kKOff + kStages * kKV;
  static constexpr int kPOff = kVOff + kStages * kKV;   // [2] P tiles
  static constexpr int kBarOff = kPOff + 2 * kP;
  static constexpr int kBytes = kBarOff + 256;
  // in-cluster merge, over the operand buffers once every MMA has finished:
  // the partial O [128 rows][DH] fp32 (16-byte chunk k of row r at k ^ (r % 8)),
  // the rows' (m, l), and per merged row the chunks' weights and 1 / L
  static constexpr int kStageOff = 0;
  static constexpr int kMlOff = kStageOff + kRows * DH * 4;
  static constexpr int kWOff = kMlOff + kRows * 8;
  static_assert(kWOff + kRows * kWStride * 4 <= kBarOff, "merge staging overlaps the barriers");
};

}  // namespace

// The in-cluster log-sum-exp merge (every thread of the CTA calls it).  The CTA of
// rank c holds key range c's partial (the cluster spans the grid's y dimension,
// so the rank is blockIdx.y).  For each of its rows [128c/C, 128(c+1)/C):
// M = max_c m_c, w_c = 2^(m_c - M) (0 for a range that saw no key),
// L = sum_c w_c l_c and o = (sum_c w_c O_c) / L, the sums in the order the merge
// kernel takes them (L as a 32-lane butterfly, O in range order), fp32 with
// every rounding explicit.
template <int DH>
__device__ __forceinline__ void attn_cluster_merge(const AttnTcArgs& a, uint8_t* smem, uint32_t sbase,
                                                   int qt, int b, int g) {
  using L = AttnSmem<DH>;
  constexpr int KC = DH / 4;          // 16-byte chunks per row
  constexpr int kU = 4;               // items whose loads are in flight together
  const int C = a.n_chunks;
  const int group = a.Hq / a.Hkv;
  const int q_rows = group * a.Tc;
  const int me = (int)attn_cluster_rank();
  const int row0 = me * kRows / C, row1 = (me + 1) * kRows / C;
  const int nrows = row1 - row0;
  float* sw = reinterpret_cast<float*>(smem + L::kWOff);
  attn_cluster_sync();                // every CTA of the cluster has staged its partial
  for (int t = threadIdx.x; t < nrows; t += blockDim.x) {
    const int r = row0 + t;
    float mc[kMaxClusterChunks], lc[kMaxClusterChunks];
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < kMaxClusterChunks; ++c) {
      mc[c] = -INFINITY;
      lc[c] = 0.f;
      if (c < C) {
        const float2 ml = attn_ld_cluster_f2(attn_mapa(sbase + L::kMlOff + (uint32_t)r * 8u, (uint32_t)c));
        mc[c] = ml.x;
        lc[c] = ml.y;
        M = fmaxf(M, ml.x);
      }
    }
    float wl[kMaxClusterChunks];
#pragma unroll
    for (int c = 0; c < kMaxClusterChunks; ++c) {
      const float w = (mc[c] == -INFINITY) ? 0.f : exp2f(__fsub_rn(mc[c], M));
      sw[t * kWStride + c] = w;
      wl[c] = __fmul_rn(w, lc[c]);
    }
    // a 32-lane xor butterfly over the ranges' w l (zero past C) adds, in lane 0,
    // ((v0 + v4) + (v2 + v6)) + ((v1 + v5) + (v3 + v7))
    const float Ls = __fadd_rn(__fadd_rn(__fadd_rn(wl[0], wl[4]), __fadd_rn(wl[2], wl[6])),
                               __fadd_rn(__fadd_rn(wl[1], wl[5]), __fadd_rn(wl[3], wl[7])));
    sw[t * kWStride + kMaxClusterChunks] = __frcp_rn(Ls);
  }
  __syncthreads();
  const int items = nrows * KC;
  for (int i0 = threadIdx.x; i0 < items; i0 += kU * (int)blockDim.x) {
    float4 acc[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < C; ++c) {
      float4 o[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int it = i0 + u * (int)blockDim.x;
        if (it < items) {
          const int r = row0 + it / KC, k = it % KC;
          o[u] = attn_ld_cluster_f4(attn_mapa(sbase + L::kStageOff + (uint32_t)r * (DH * 4) +
                                                  (uint32_t)((k ^ (r & 7)) * 16),
                                              (uint32_t)c));
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int it = i0 + u * (int)blockDim.x;
        if (it < items) {
          const float w = sw[(it / KC) * kWStride + c];
          acc[u].x = __fmaf_rn(w, o[u].x, acc[u].x);
          acc[u].y = __fmaf_rn(w, o[u].y, acc[u].y);
          acc[u].z = __fmaf_rn(w, o[u].z, acc[u].z);
          acc[u].w = __fmaf_rn(w, o[u].w, acc[u].w);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int it = i0 + u * (int)blockDim.x;
      if (it >= items) continue;
      const int rr = it / KC, k = it % KC;
      const int qr = qt * kRows + row0 + rr;
      if (qr >= q_rows) continue;
      const int h = g * group + qr / a.Tc, i = qr % a.Tc;
      const float inv = sw[rr * kWStride + kMaxClusterChunks];
      const __nv_bfloat162 lo = __floats2bfloat162_rn(__fmul_rn(acc[u].x, inv), __fmul_rn(acc[u].y, inv));
      const __nv_bfloat162 hi = __floats2bfloat162_rn(__fmul_rn(acc[u].z, inv), __fmul_rn(acc[u].w, inv));
      bf16* dst = a.out + ((size_t)b * a.Tc + i) * ((size_t)a.Hq * DH) + (size_t)h * DH + 4 * k;
      *reinterpret_cast<uint2*>(dst) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
    }
  }
  attn_cluster_sync();                // no CTA leaves while a peer still reads it
}

template <int DH>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapKc,
               const __grid_constant__ CUtensorMap mapVc, const __grid_constant__ CUtensorMap mapKp,
               const __grid_constant__ CUtensorMap mapVp, const __grid_constant__ CUtensorMap mapPo,
               const AttnTcArgs a) {
  using L = AttnSmem<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + L::kBarOff;
  // barrier slots (8 bytes each)
  const uint32_t q_full = bars + 0;
  // K and V of a block have rings of their own: K(j) is released as soon as
  // QK^T(j) has read it, V(j) after PV(j), so each load is issued about two
  // blocks before it is used
  auto k_full = [&](int s) { return bars + 8u * (1 + s); };
  auto k_empty = [&](int s) { return bars + 8u * (3 + s); };
  auto v_full = [&](int s) { return bars + 8u * (13 + s); };
  auto v_empty = [&](int s) { return bars + 8u * (15 + s); };
  auto s_full = [&](int s) { return bars + 8u * (5 + s); };
  auto s_free = [&](int s) { return bars + 8u * (7 + s); };
  auto p_full = [&](int b) { return bars + 8u * (9 + b); };     // P tile b written
  auto pv_done = [&](int b) { return bars + 8u * (11 + b); };   // the PV MMAs reading P tile b done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBarOff + 8 * 17);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kBarOff + 8 * 17 + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, chunk = blockIdx.y;
  const int b = blockIdx.z / a.Hkv, g = blockIdx.z % a.Hkv;
  const int group = a.Hq / a.Hkv;
  const int q_rows = group * a.Tc;
  const int nbp = (a.n_vis + kBN - 1) / kBN;            // prompt-key blocks
  const int nbc = (a.Tc + kBN - 1) / kBN;               // canvas-key blocks
  const int nb = nbp + nbc;
  // Key blocks this query tile needs: all of them, or in causal mode those that
  // meet some row's visible positions [P + i - window + 1, P + i] (the tile's rows
  // are new tokens i_min .. i_max, or every i when the tile crosses a head).
  int js = 0, je = nb;
  if (a.causal) {
    const int r0 = qt * kRows, r1 = min(r0 + kRows, q_rows) - 1;
    const int i_min = (r0 / a.Tc == r1 / a.Tc) ? r0 % a.Tc : 0;
    const int i_max = (r0 / a.Tc == r1 / a.Tc) ? r1 % a.Tc : a.Tc - 1;
    je = nbp + i_max / kBN + 1;
    if (a.window > 0) {
      const int lo = a.P + i_min - a.window + 1;        // lowest position a row sees
      const int first = a.P - a.n_vis;                  // position of prompt block 0, key 0
      js = (lo < a.P) ? max(0, lo - first) / kBN : nbp + (lo - a.P) / kBN;
    }
  }
  const int jb0 = js + (int)(((long long)chunk * (je - js)) / a.n_chunks);
  const int jb1 = js + (int)(((long long)(chunk + 1) * (je - js)) / a.n_chunks);
  const int n_local = jb1 - jb0;
  // TMEM: O at [0, DH); then two S buffers (the next QK^T runs while the
  // softmax reads the last one), each split into two independent accumulator
  // chains of kBN columns: the k16 steps of QK^T alternate between them, so
  // consecutive MMAs do not wait for one another.
  constexpr int kSChains = 2;
  constexpr int kSBufs = 2;
  constexpr uint32_t kTmemCols = (DH + kSBufs * kSChains * kBN <= 256) ? 256 : 512;
  constexpr uint32_t kOCol = 0, kSCol = DH;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
      mbar_init(s_full(s), 1);
      mbar_init(s_free(s), 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(p_full(b), 4);
      mbar_init(pv_done(b), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapKc);
    tma_prefetch_desc(&mapVc);
    tma_prefetch_desc(&mapKp);
    tma_prefetch_desc(&mapVp);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The prompt K/V is set before the pass and never written by it: the
  // producer issues the first ring stages of prompt blocks before the grid
  // wait (fresh barriers, no empty waits); q and the canvas K/V come after it.
  auto block_src = [&](int j, const CUtensorMap*& mk, const CUtensorMap*& mv, int& row) {
    const int jg = jb0 + j;
    if (jg < nbp) {
      mk = &mapKp; mv = &mapVp;
      row = (b * a.Hkv + g) * a.kv_stride + (a.P - a.n_vis) + jg * kBN;
    } else {
      mk = &mapKc; mv = &mapVc;
      row = (b * a.Hkv + g) * a.Tc + (jg - nbp) * kBN;
    }
  };
  auto issue_k = [&](int j) {
    const int st = j % kStages;
    const CUtensorMap *mk, *mv;
    int row;
    block_src(j, mk, mv, row);
    mbar_arrive_expect_tx(k_full(st), (uint32_t)L::kKV);
    for (int c = 0; c < DH / 64; ++c)
      tma_load_2d(sbase + L::kKOff + st * L::kKV + c * (kBN * 128), mk, k_full(st), c * 64, row);
  };
  auto issue_v = [&](int j) {
    const int st = j % kStages;
    const CUtensorMap *mk, *mv;
    int row;
    block_src(j, mk, mv, row);
    mbar_arrive_expect_tx(v_full(st), (uint32_t)L::kKV);
    for (int c = 0; c < DH / 64; ++c)
      tma_load_2d(sbase + L::kVOff + st * L::kKV + c * (kBN * 128), mv, v_full(st), c * 64, row);
  };
  int pre_kv = 0;
  if (warp == 0 && lane == 0)
    while (pre_kv < kStages && pre_kv < n_local && jb0 + pre_kv < nbp) {
      issue_k(pre_kv);
      issue_v(pre_kv);
      ++pre_kv;
    }
  griddep_wait();
  griddep_launch();

  if (warp == 0) {
    if (lane == 0 && n_local > 0) {
      // ---------------------------------------------------------- TMA producer
      const int q_row0 = (b * a.Hq + g * group) * a.Tc + qt * kRows;
      mbar_arrive_expect_tx(q_full, (uint32_t)L::kQ);
      for (int c = 0; c < DH / 64; ++c)
        tma_load_2d(sbase + L::kQOff + c * (kRows * 128), &mapQ, q_full, c * 64, q_row0);
      bool ok = true;
      // K(j) waits for QK^T(j - 2), V(j) for PV(j - 2); V is issued one block
      // behind K, which is the order in which the MMAs free their stages
      int ik = pre_kv, iv = pre_kv;
      while (ok && (ik < n_local || iv < n_local)) {
        if (ik < n_local) {
          if (!mbar_wait(k_empty(ik % kStages), (uint32_t)((ik / kStages) & 1) ^ 1u, abort_flag, a.err)) {
            ok = false;
            break;
          }
          issue_k(ik++);
        }
        if (iv < n_local && (iv < ik - 1 || ik == n_local)) {
          if (!mbar_wait(v_empty(iv % kStages), (uint32_t)((iv / kStages) & 1) ^ 1u, abort_flag, a.err)) {
            ok = false;
            break;
          }
          issue_v(iv++);
        }
      }
      if (!ok) {  // abort path: let issued copies land
        mbar_drain(q_full, 0);
        for (int j = (ik > kStages ? ik - kStages : 0); j < ik; ++j)
          mbar_drain(k_full(j % kStages), (uint32_t)((j / kStages) & 1));
        for (int j = (iv > kStages ? iv - kStages : 0); j < iv; ++j)
          mbar_drain(v_full(j % kStages), (uint32_t)((j / kStages) & 1));
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && n_local > 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t idesc_s = idesc_bf16_f32(kBN);
      const uint32_t idesc_o = idesc_bf16_f32(DH, false, true);   // B (= V) MN-major
      bool ok = mbar_wait(q_full, 0, abort_flag, a.err);
      tc_fence_after();
      for (int j = 0; j <= n_local && ok; ++j) {
        if (j < n_local) {
          const int st = j % kStages, sb = j % kSBufs;
          if (!mbar_wait(k_full(st), (uint32_t)((j / kStages) & 1), abort_flag, a.err)) { ok = false; break; }
          if (!mbar_wait(s_free(sb), (uint32_t)((j / kSBufs) & 1) ^ 1u, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kbase = sbase + L::kKOff + st * L::kKV;
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            const int c = kk >> 2, w = (kk & 3) * 32;
            const int ch = kk % kSChains;
            const uint64_t ad = sdesc_kmajor_sw128(sbase + L::kQOff + c * (kRows * 128) + w);
            const uint64_t bd = sdesc_kmajor_sw128(kbase + c * (kBN * 128) + w);
            umma_bf16(tmem + kSCol + (sb * kSChains + ch) * kBN, ad, bd, idesc_s,
                      kk >= kSChains ? 1u : 0u);
          }
          umma_commit(s_full(sb));
          umma_commit(k_empty(st));
        }
        if (j >= 1) {
          const int jp = j - 1, stp = jp % kStages;
          if (!mbar_wait(p_full(jp & 1), (uint32_t)((jp >> 1) & 1), abort_flag, a.err)) { ok = false; break; }
          if (!mbar_wait(v_full(stp), (uint32_t)((jp / kStages) & 1), abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t vbase = sbase + L::kVOff + stp * L::kKV;
          const uint32_t pbase = sbase + L::kPOff + (uint32_t)(jp & 1) * L::kP;
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint64_t ad = sdesc_kmajor_sw128(pbase + kk * 32);
            const uint64_t bd = sdesc_mnmajor_sw128(vbase + kk * (16 * 128), kBN * 128);
            umma_bf16(tmem + kOCol, ad, bd, idesc_o, (jp > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(pv_done(jp & 1));
          umma_commit(v_empty(stp));
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int q = warp & 3;
    const int r = q * 32 + lane;                       // query row in the tile
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    // causal mode: this row's new-token index i and its visible positions
    // [lo_pos, P + i] (keys are numbered by position: cached ones from P - n_vis)
    const int i_row = (qt * kRows + r) % a.Tc;
    const int hi_pos = a.P + i_row;
    const int lo_pos = a.window > 0 ? hi_pos - a.window + 1 : INT_MIN;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    uint32_t v[32];
    for (int j = 0; j < n_local; ++j) {
      const int sb = j % kSBufs;
      // waits are made warp-uniform: the warp-wide votes and tcgen05 loads below
      // need every lane, also on the abort path
      if (!__all_sync(0xffffffffu, mbar_wait(s_full(sb), (uint32_t)((j / kSBufs) & 1), abort_flag, a.err))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kBN];
#pragma unroll
      for (int h = 0; h < kBN / 32; ++h) {
        // chains summed in a fixed order: ((c0 + c1) + c2) + c3, two loads per wait
        uint32_t v2[32];
#pragma unroll
        for (int ch = 0; ch < kSChains; ch += 2) {
          tmem_ld32(lane_base + kSCol + (sb * kSChains + ch) * kBN + h * 32, v);
          tmem_ld32(lane_base + kSCol + (sb * kSChains + ch + 1) * kBN + h * 32, v2);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float x = (ch == 0) ? __uint_as_float(v[e]) : s[h * 32 + e] + __uint_as_float(v[e]);
            s[h * 32 + e] = x + __uint_as_float(v2[e]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free(sb));
      // mask and scale
      const int jg = jb0 + j;
      const int valid = (jg < nbp) ? min(kBN, a.n_vis - jg * kBN) : min(kBN, a.Tc - (jg - nbp) * kBN);
      float bmax = -INFINITY;
      if (a.causal) {
        const int pos0 = (jg < nbp) ? a.P - a.n_vis + jg * kBN : a.P + (jg - nbp) * kBN;
#pragma unroll
        for (int e = 0; e < kBN; ++e) {
          const bool vis = e < valid && pos0 + e <= hi_pos && pos0 + e >= lo_pos;
          s[e] = vis ? s[e] * a.scale_log2 : -INFINITY;
          bmax = fmaxf(bmax, s[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < kBN; ++e) {
          s[e] = (e < valid) ? s[e] * a.scale_log2 : -INFINITY;
          bmax = fmaxf(bmax, s[e]);
        }
      }
      // A row whose block max passes its reference max by the threshold rescales
      // O; tcgen05.ld/st are warp-wide, so the warp rescales when any lane must
      // (factor 1 for the others), after every PV so far has finished.  Without
      // a rescale, P_j only needs its buffer back: PV_{j-2} done.
      const bool grow = m != -INFINITY && bmax > m + kRescaleThreshold;
      const bool rescale = __any_sync(0xffffffffu, grow);
      if (rescale && j >= 1) {
        if (!__all_sync(0xffffffffu, mbar_wait(pv_done((j - 1) & 1), (uint32_t)(((j - 1) >> 1) & 1),
                                                abort_flag, a.err))) { ok = false; break; }
        tc_fence_after();
      } else if (j >= 2) {
        if (!__all_sync(0xffffffffu, mbar_wait(pv_done(j & 1), (uint32_t)(((j - 2) >> 1) & 1),
                                                abort_flag, a.err))) { ok = false; break; }
        tc_fence_after();
      }
      if (rescale) {
        const float f = grow ? exp2f(m - bmax) : 1.0f;
#pragma unroll 1
        for (int c0 = 0; c0 < DH; c0 += 32) {
          tmem_ld32(lane_base + kOCol + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
          tmem_st32(lane_base + kOCol + c0, v);
        }
        tmem_wait_st();
        l *= f;
      }
      if (m == -INFINITY || grow) m = bmax;
      // P = 2^(s - m) as bf16, row r of the K-major swizzled tile (a row that has
      // seen no visible key yet, possible in causal mode, writes zeros)
      const float msub = (m == -INFINITY) ? 0.f : m;
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int e = 0; e < kBN; e += 2) {
        const float p0 = exp2f(s[e] - msub), p1 = exp2f(s[e + 1] - msub);
        l += p0 + p1;
        __nv_bfloat162 bb = __floats2bfloat162_rn(p0, p1);
        pk[e / 2] = *reinterpret_cast<uint32_t*>(&bb);
      }
      uint8_t* prow = smem + L::kPOff + (j & 1) * L::kP + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int pc = c ^ (r & 7);
        *reinterpret_cast<uint4*>(prow + pc * 16) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full(j & 1));
    }
    // final O, then the partial of this key range
    if (ok && n_local > 0)
      ok = mbar_wait(pv_done((n_local - 1) & 1), (uint32_t)(((n_local - 1) >> 1) & 1), abort_flag, a.err);
    tc_fence_after();
    if (a.fused) {
      // stage the partial for the cluster's merge: this thread's row r, 32 columns per
      // TMEM load, 16-byte chunk k at k ^ (r % 8) (eight consecutive rows cover all banks)
      const uint32_t srow = sbase + L::kStageOff + (uint32_t)r * (DH * 4);
#pragma unroll 1
      for (int c0 = 0; c0 < DH; c0 += 32) {
        if (n_local > 0 && ok) {
          tmem_ld32(lane_base + kOCol + c0, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4)
          st_shared_v4(srow + (uint32_t)((((c0 >> 2) + c4) ^ (r & 7)) * 16), v[4 * c4], v[4 * c4 + 1],
                       v[4 * c4 + 2], v[4 * c4 + 3]);
      }
      reinterpret_cast<float2*>(smem + L::kMlOff)[r] = make_float2((n_local > 0) ? m : -INFINITY, l);
    } else {
    const int qr = qt * kRows + r;
    const int rows_total = a.B * a.Hq * a.Tc;
    const bool row_valid = qr < q_rows;
    size_t R = 0;
    if (row_valid) {
      const int h = g * group + qr / a.Tc, i = qr % a.Tc;
      R = ((size_t)b * a.Hq + h) * a.Tc + i;
    }
    float* po = a.part_o + ((size_t)chunk * rows_total + R) * DH;
    // The partial O leaves through shared memory: this warp stages its 32 rows
    // x 32 columns (128-byte swizzle: float4 c of row r at c ^ (r % 8)) in the
    // K/V ring, idle now, and lane 0 writes the block with a tensor store.
    // The 32 rows are consecutive in part_o when all are valid (R = R0 + qr);
    // otherwise the valid ones are written directly.
    const bool warp_full = __all_sync(0xffffffffu, row_valid);
    const int row0 = chunk * rows_total + (b * a.Hq + g * group) * a.Tc + qt * kRows + q * 32;
    const uint32_t stage_base = sbase + L::kKOff + (uint32_t)(warp - 2) * 8192u;
#pragma unroll 1
    for (int c0 = 0, sbuf = 0; c0 < DH; c0 += 32, sbuf ^= 1) {
      if (n_local > 0 && ok) {
        tmem_ld32(lane_base + kOCol + c0, v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if (warp_full) {
        const uint32_t st = stage_base + (uint32_t)sbuf * 4096u;
        if (lane == 0) bulk_wait_read<1>();   // the store that last read this buffer is done
        __syncwarp();
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4)
          st_shared_v4(st + (uint32_t)lane * 128u + (uint32_t)((c4 ^ (lane & 7)) * 16),
                       v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&mapPo, st, c0, row0);
          bulk_commit();
        }
      } else if (row_valid) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(po + c0 + e) =
              make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                          __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
      }
    }
    if (warp_full && lane == 0) bulk_wait_all();
    __syncwarp();
    if (row_valid) {
      float* pml = a.part_ml + ((size_t)chunk * rows_total + R) * 2;
      pml[0] = (n_local > 0) ? m : -INFINITY;
      pml[1] = l;
    }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  // every thread of every CTA reaches this point on every path (no early exit), so
  // the cluster barriers inside always complete
  if (a.fused) attn_cluster_merge<DH>(a, smem, sbase, qt, b, g);
}

namespace {

template <int DH>
cudaError_t launch_attn_tc_t(const AttnTcMaps& m, const AttnTcArgs& a, cudaStream_t s) {
  const size_t smem = AttnSmem<DH>::kBytes + 1024;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(attn_tc_kernel<DH>), (int)smem);
  if (e != cudaSuccess) return e;
  const int group = a.Hq / a.Hkv;
  dim3 grid((group * a.Tc + kRows - 1) / kRows, a.n_chunks, a.B * a.Hkv);
  if (!a.fused)
    return launch_k(attn_tc_kernel<DH>, grid, dim3(kThreads), smem, s, m.q, m.kc, m.vc, m.kp, m.vp,
                    m.po, a);
  if (a.n_chunks < 1 || a.n_chunks > kMaxClusterChunks || a.out == nullptr) return cudaErrorInvalidValue;
  // the key ranges of one query tile form one cluster along y
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = (unsigned)a.n_chunks;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, attn_tc_kernel<DH>, m.q, m.kc, m.vc, m.kp, m.vp, m.po, a);
}

template <int DH>
int attn_fused_clusters_t(int n_chunks) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, (unsigned)n_chunks, 1);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = AttnSmem<DH>::kBytes + 1024;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = (unsigned)n_chunks;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (ensure_smem_limit(reinterpret_cast<const void*>(attn_tc_kernel<DH>),
                        (int)(AttnSmem<DH>::kBytes + 1024)) != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel<DH>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  return n;
}

}  // namespace

bool attn_tc_fused_ok(int dh, int n_chunks) {
  if (n_chunks < 1 || n_chunks > kMaxClusterChunks) return false;
  static std::mutex mu;
  static std::map<std::tuple<int, int, int>, int> cache;   // (device, dh, chunks) -> clusters
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_tuple(dev, dh, n_chunks);
  auto it = cache.find(key);
  if (it == cache.end()) {
    int n = 0;
    switch (dh) {
      case 64: n = attn_fused_clusters_t<64>(n_chunks); break;
      case 128: n = attn_fused_clusters_t<128>(n_chunks); break;
      case 256: n = attn_fused_clusters_t<256>(n_chunks); break;
      default: n = 0;
    }
    it = cache.emplace(key, n).first;
  }
  return it->second > 0;
}

int attn_tc_blocks(int n_vis, int Tc) { return (n_vis + kBN - 1) / kBN + (Tc + kBN - 1) / kBN; }
int attn_tc_qtiles(int Hq, int Hkv, int Tc) { return (Hq / Hkv * Tc + kRows - 1) / kRows; }

cudaError_t launch_attention_tc(const AttnTcMaps& m, const AttnTcArgs& a, cudaStream_t s) {
  switch (a.dh) {
    case 64: return launch_attn_tc_t<64>(m, a, s);
    case 128: return launch_attn_tc_t<128>(m, a, s);
    case 256: return launch_attn_tc_t<256>(m, a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dg
