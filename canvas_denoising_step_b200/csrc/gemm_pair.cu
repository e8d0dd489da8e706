// Two-SM tcgen05 GEMM (cta_group::2) for the dense projections and the
// expert gate/up and down GEMMs.
//
// A cluster of two CTAs on neighbouring SMs computes one tile pair: CTA r
// holds weight slab 2p + r (128 rows, the A operand) and half of the tile's
// N activation rows (the B operand), and the leader CTA (rank 0) issues
// tcgen05.mma with M = 256 over both CTAs' shared memory.  Each CTA then owns
// a 128 x N fp32 accumulator in its own TMEM and runs the one-SM engine's
// epilogue on it.  Against two one-SM tiles, every SM takes in half of the
// activation bytes per k-block (the pair reads the activation tile once, not
// once per slab); at N = 256 a one-SM tile streams two activation bytes (from
// L2) per weight byte (from HBM), and that ingest is what bounds these GEMMs.
//
// Roles (192 threads per CTA):
//   warp 0 lane 0   TMA producer in both CTAs; every load signals the
//                   leader's "full" barrier of its k-block (cta_group::2
//                   form).  In the grouped modes the leader's producer also
//                   takes tile pairs from the counter and publishes each to
//                   both CTAs' tile queues.
//   warp 1          TMEM allocation (both CTAs, cta_group::2); lane 0 of the
//                   leader issues the MMAs and commits to both CTAs' "empty"
//                   and "tmem full" barriers
//   warps 2..5      epilogue of the CTA's own accumulator rows; each warp
//                   arrives on the leader's "tmem empty" barrier (count 8)
// The operand ring is byte-addressed as in the one-SM engine (a k-block takes
// its weight tile and its B boxes, never wraps, at most kPairSlots in
// flight); both CTAs walk the same tile sequence and place blocks alike, so
// the leader's descriptors address the same offsets in both.
// The dense projections deal tile pairs statically (cluster p takes p,
// p + clusters, ...); the grouped modes longest chunk first from a counter.
// Every wait is bounded (kWaitLimitNs); both CTAs meet at a cluster barrier
// before either frees TMEM or exits, so no CTA leaves while its peer can
// still reach its shared memory.
#include <map>
#include <mutex>

#include "gemm_shared.cuh"

namespace dg {

namespace {

constexpr int kPairThreads = 192;
constexpr int kPairSlots = 16;   // barrier slots of the operand ring

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address, in the cluster's shared window, of this CTA's shared variable at
// `addr` as it sits in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Arrive on an mbarrier of another CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

// Tensor load into this CTA's shared memory whose bytes count on an mbarrier
// of either CTA of the pair (bar: a cluster-window address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Store a 32-bit word into the shared memory of a CTA of the cluster.
__device__ __forceinline__ void st_cluster_b32(uint32_t cluster_addr, int v) {
  asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// Parity wait whose acquire covers writes that another CTA of the cluster
// released (bounded like mbar_wait).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity,
                                                  volatile int* abort, int* err) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (*abort) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort = 1;
      raise_error(err, kErrTimeout);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D (+)= A * B^T over the CTA pair: M = 256 (128 A rows from each CTA's shared
// memory at the descriptor's offset), N B rows (N/2 from each CTA).
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier at a cluster-window address when this thread's
// earlier pair MMAs have completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t cluster_bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   cluster_bar)
               : "memory");
}

// Instruction descriptor of the pair MMA: bf16 x bf16 -> fp32, M = 256, N = n.
__device__ __forceinline__ uint32_t idesc_pair(int n) {
  return (idesc_bf16_f32(n) & ~(0x1Fu << 24)) | ((uint32_t)(256 >> 4) << 24);
}

}  // namespace

__global__ void __launch_bounds__(kPairThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                 const __grid_constant__ CUtensorMap mapC, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  constexpr int S = kPairSlots;
  const int max_inflight = a.stages;            // k-blocks in flight at most (<= S)
  const uint32_t cap = (uint32_t)a.ring_bytes;  // operand ring bytes
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)a.ring_bytes);
  // full[0..S) (the leader's count both CTAs' bytes), empty[S..2S),
  // tmem_full[2S..2S+2), tmem_empty[2S+2..2S+4) (the leader's count 8 warps),
  // tile queue full / empty [2S+4 .. 2S+4+2*kTileQ)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4 + 2 * kTileQ);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_tq = reinterpret_cast<volatile int*>(tmem_slot + 2);   // [kTileQ] tile pairs
  uint32_t* s_vstart = tmem_slot + 2 + kTileQ;   // [S] running ring start of each slot's block
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_u32(bars);
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (S + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * S + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * S + 2 + b); };
  auto tq_full_bar = [&](int q) { return bar_base + 8u * (2 * S + 4 + q); };
  auto tq_empty_bar = [&](int q) { return bar_base + 8u * (2 * S + 4 + kTileQ + q); };

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const uint32_t peer = rank ^ 1u;
  const bool grouped = a.mode == GEMM_GATEUP || a.mode == GEMM_DOWN;
  const bool dyn = grouped && a.tile_counter != nullptr;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 8);   // four epilogue warps in each CTA
    }
    for (int q = 0; q < kTileQ; ++q) {
      mbar_init(tq_full_bar(q), 1);
      // the leader's MMA lane and epilogue warps, the peer's producer and
      // epilogue warps
      mbar_init(tq_empty_bar(q), 10);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  // both CTAs' barriers are initialised and TMEM allocated before either
  // signals the other
  tc_fence_before();
  cluster_barrier();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Group tables (grouped modes): written by the router, which had completed
  // before the kernel just before this one let it launch (each of the router,
  // the row gather and the gate/up GEMM triggers its dependents only after its
  // own grid wait), so they are read before this kernel's wait.
  int* s_prefix = reinterpret_cast<int*>(smem + (size_t)a.ring_bytes + 1024);
  int* s_offsets = s_prefix + (a.n_groups + 1);
  int* s_order = (grouped && a.chunk_order) ? s_offsets + (a.n_groups + 1) : nullptr;
  float* s_stage_out = reinterpret_cast<float*>(smem + (size_t)a.ring_bytes + 1024 + a.tab_bytes);
  if (grouped) {
    for (int i = threadIdx.x; i <= a.n_groups; i += blockDim.x) {
      s_prefix[i] = __ldcg(a.chunk_prefix + i);
      s_offsets[i] = __ldcg(a.offsets + i);
    }
    __syncthreads();
    if (s_order)
      for (int i = threadIdx.x; i < s_prefix[a.n_groups]; i += blockDim.x)
        s_order[i] = __ldcg(a.chunk_order + i);
    __syncthreads();
  }
  // A DOWN launch with ready counters does not wait for the whole gate/up
  // grid: its H rows are guarded per chunk below.
  const bool handover = a.mode == GEMM_DOWN && a.chunk_ready != nullptr;
  if (!handover) griddep_wait();
  griddep_launch();

  // Tile pair pt = (activation chunk / split, slab pair sp): this CTA's tile
  // has weight slab 2 sp + rank (m_slabs is even), the same rows, chunk and
  // split in both CTAs.
  const int half = a.m_slabs / 2;
  const int n_pt = tile_count(a, grouped ? s_prefix : nullptr) / 2;
  const int cl = blockIdx.x >> 1, n_cl = gridDim.x >> 1;
  auto own_tile = [&](int pt) { return (pt / half) * a.m_slabs + 2 * (pt % half) + (int)rank; };
  // B rows this CTA supplies (half of the MMA's N) and their boxes
  auto b_half = [&](const TileInfo& ti) { return ti.n_mma / 2; };
  auto b_boxes = [&](const TileInfo& ti) { return (b_half(ti) + a.b_box_rows - 1) / a.b_box_rows; };
  auto blk_size = [&](const TileInfo& ti) -> uint32_t {
    return (uint32_t)kATileBytes + (uint32_t)(b_boxes(ti) * a.b_box_rows * 128);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int j = 0, tail = 0;           // k-blocks placed; oldest block not yet retired
      uint32_t vpos = 0, roff = 0;   // ring position: running (never wraps) and offset
      bool ok = true;
      for (int it = 0; ok; ++it) {
        int pt;
        if (dyn) {
          const int q = it % kTileQ;
          const uint32_t par = (uint32_t)((it / kTileQ) & 1);
          if (leader) {
            // take the next tile pair and publish it to both CTAs
            if (!mbar_wait(tq_empty_bar(q), par ^ 1u, abort_flag, a.err)) { ok = false; break; }
            pt = atomicAdd(a.tile_counter, 1);
            if (pt >= n_pt) pt = -1;
            s_tq[q] = pt;
            st_cluster_b32(mapa_rank(smem_u32((const void*)(s_tq + q)), peer), pt);
            mbar_arrive(tq_full_bar(q));
            mbar_arrive_remote(mapa_rank(tq_full_bar(q), peer));
          } else {
            if (!mbar_wait_cluster(tq_full_bar(q), par, abort_flag, a.err)) { ok = false; break; }
            pt = s_tq[q];
            mbar_arrive_remote(mapa_rank(tq_empty_bar(q), 0));
          }
          if (pt < 0) break;
        } else {
          pt = cl + it * n_cl;
          if (pt >= n_pt) break;
        }
        const TileInfo ti = decode_tile(a, own_tile(pt), s_prefix, s_offsets, s_order);
        const int nh = b_half(ti), nb = b_boxes(ti);
        const uint32_t blk = blk_size(ti);
        if (handover) {
          // this chunk's H rows are written by every gate/up slab's epilogue
          const int* rc = a.chunk_ready + ti.chunk;
          const unsigned long long t0 = globaltimer_ns();
          while (ld_acquire(rc) < a.ready_target) {
            if (*abort_flag || globaltimer_ns() - t0 > kWaitLimitNs) {
              *abort_flag = 1;
              raise_error(a.err, kErrTimeout);
              ok = false;
              break;
            }
          }
          if (!ok) break;
          fence_proxy_async_global();   // the TMA loads below see those writes
        }
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++j) {
          if (roff + blk > cap) { vpos += cap - roff; roff = 0; }
          const uint32_t sA = smem_base + roff;
          const uint32_t sB = sA + (uint32_t)kATileBytes;
          const int slot = j % S;
          // retire the oldest blocks until this one's bytes and slot are free:
          // the blocks in flight span [start of the oldest, vpos + blk) of the
          // running position, which must fit in the ring
          while (tail < j && (j - tail >= max_inflight || s_vstart[tail % S] + cap < vpos + blk)) {
            if (!mbar_wait(empty_bar(tail % S), (uint32_t)((tail / S) & 1), abort_flag, a.err)) {
              ok = false;
              break;
            }
            ++tail;
          }
          if (!ok) break;
          if (leader) mbar_arrive_expect_tx(full_bar(slot), 2u * blk);
          s_vstart[slot] = vpos;
          vpos += blk;
          roff += blk;
          const uint32_t fb = mapa_rank(full_bar(slot), 0);
          const int kx = kb * kBK;
          if (grouped) tma_load_3d_pair(sA, &mapA, fb, kx, ti.a_row0, ti.g);
          else tma_load_2d_pair(sA, &mapA, fb, kx, ti.a_row0);
          for (int i = 0; i < nb; ++i)
            tma_load_2d_pair(sB + (uint32_t)(i * a.b_box_rows * 128), &mapB, fb, kx,
                             ti.row0 + (int)rank * nh + i * a.b_box_rows);
        }
      }
      if (!ok && leader) {
        // abort path: blocks still in flight (both CTAs' bytes count here)
        // land before the pair meets at the final barrier
        for (int i = tail; i < j; ++i) mbar_drain(full_bar(i % S), (uint32_t)((i / S) & 1));
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer
      int j = 0;
      uint32_t roff = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        int pt;
        if (dyn) {
          const int q = it % kTileQ;
          if (!mbar_wait(tq_full_bar(q), (uint32_t)((it / kTileQ) & 1), abort_flag, a.err)) break;
          pt = s_tq[q];
          mbar_arrive(tq_empty_bar(q));
          if (pt < 0) break;
        } else {
          pt = cl + it * n_cl;
          if (pt >= n_pt) break;
        }
        const TileInfo ti = decode_tile(a, own_tile(pt), s_prefix, s_offsets, s_order);
        const uint32_t blk = blk_size(ti);
        const int buf = it & 1;
        const uint32_t tph = (uint32_t)((it >> 1) & 1);
        if (!mbar_wait(tempty_bar(buf), tph ^ 1u, abort_flag, a.err)) break;
        tc_fence_after();
        const uint32_t d_base = tmem_base + (uint32_t)buf * kAccCols;
        const uint32_t idesc = idesc_pair(ti.n_mma);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++j) {
          if (roff + blk > cap) roff = 0;
          const int slot = j % S;
          if (!mbar_wait(full_bar(slot), (uint32_t)((j / S) & 1), abort_flag, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_base + roff;
          const uint32_t sB = sA + (uint32_t)kATileBytes;
          roff += blk;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_bf16_pair(d_base, sdesc_kmajor_sw128(sA + kk * 32),
                           sdesc_kmajor_sw128(sB + kk * 32), idesc,
                           (kb > ti.kb0 || kk > 0) ? 1u : 0u);
          umma_commit_pair(mapa_rank(empty_bar(slot), 0));
          umma_commit_pair(mapa_rank(empty_bar(slot), 1));
        }
        if (!ok) break;
        umma_commit_pair(mapa_rank(tfull_bar(buf), 0));
        umma_commit_pair(mapa_rank(tfull_bar(buf), 1));
      }
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int n_sbuf = a.epi_bytes / (4 * 4096);
    float* s_warp_out = s_stage_out + (warp - 2) * n_sbuf * 1024;
    int sbuf = 0;
    for (int it = 0;; ++it) {
      int pt;
      if (dyn) {
        const int qi = it % kTileQ;
        const uint32_t par = (uint32_t)((it / kTileQ) & 1);
        const bool got = leader ? mbar_wait(tq_full_bar(qi), par, abort_flag, a.err)
                                : mbar_wait_cluster(tq_full_bar(qi), par, abort_flag, a.err);
        if (!got) break;
        pt = s_tq[qi];
        __syncwarp();
        if (lane == 0) {
          if (leader) mbar_arrive(tq_empty_bar(qi));
          else mbar_arrive_remote(mapa_rank(tq_empty_bar(qi), 0));
        }
        if (pt < 0) break;
      } else {
        pt = cl + it * n_cl;
        if (pt >= n_pt) break;
      }
      const TileInfo ti = decode_tile(a, own_tile(pt), s_prefix, s_offsets, s_order);
      const int buf = it & 1;
      const uint32_t tph = (uint32_t)((it >> 1) & 1);
      if (!mbar_wait(tfull_bar(buf), tph, abort_flag, a.err)) break;
      tc_fence_after();
      const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)buf * kAccCols;
      if (a.mode == GEMM_GATEUP)
        epi_gateup_tile(a, &mapC, ti, lane_addr, q, lane,
                        smem_u32(s_stage_out) + (uint32_t)(warp - 2) * 2048u, sbuf, nullptr);
      else
        epi_f32_tile(a, &mapC, ti, lane_addr, q, lane, s_warp_out, n_sbuf, sbuf, nullptr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(tempty_bar(buf));
        else mbar_arrive_remote(mapa_rank(tempty_bar(buf), 0));
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_barrier();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// Shared-memory plan of the pair GEMM: the operand ring takes what the barriers,
// group tables and output staging leave.  A k-block is the CTA's 16 KB weight
// tile plus its B boxes (half of the tile's activation rows); the dense
// projections keep at most 8 in flight, the grouped modes are bound by bytes.
void gemm_pair_plan_smem(GemmArgs& a) {
  const bool grouped = a.mode == GEMM_GATEUP || a.mode == GEMM_DOWN;
  a.n_bufs = 2;
  a.pair = 0;
  a.dense_pair = 0;
  a.tab_bytes = grouped ? ((2 * (a.n_groups + 1) * 4 + (a.chunk_order ? a.max_chunks * 4 : 0) +
                            127) / 128) * 128 : 0;
  a.epi_bytes = a.mode == GEMM_GATEUP ? 2 * 4 * 1024 : (a.mode == GEMM_DOWN ? 4 * 4096 : 2 * 4 * 4096);
  a.a_bytes = kATileBytes;
  const int half_rows = (a.n_tile + 1) / 2;
  a.b_bytes = ((half_rows + a.b_box_rows - 1) / a.b_box_rows) * a.b_box_rows * 128;
  a.stage_bytes = a.a_bytes + a.b_bytes;
  a.ring_bytes = ((kMaxSmem - 2048 - a.tab_bytes - a.epi_bytes) / 1024) * 1024;
  if (a.ring_bytes < 2 * a.stage_bytes) a.ring_bytes = 2 * a.stage_bytes;  // launch refuses
  const int s = a.ring_bytes / a.stage_bytes;
  a.stages = grouped ? kPairSlots : (s > 8 ? 8 : s);
}

size_t gemm_pair_smem_bytes(const GemmArgs& a) {
  return 1024 + (size_t)a.ring_bytes + 1024 + a.tab_bytes + a.epi_bytes;
}

int gemm_pair_max_clusters() {
  // per device, as the occupancy it answers
  static std::mutex mu;
  static std::map<int, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(dev);
  if (it == cache.end()) {
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kPairThreads);
    cfg.dynamicSmemBytes = kMaxSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (ensure_smem_limit(reinterpret_cast<const void*>(gemm_pair_kernel), kMaxSmem) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    it = cache.emplace(dev, n).first;
  }
  return it->second;
}

cudaError_t gemm_pair_launch(const CUtensorMap& mapA, const CUtensorMap& mapB_half,
                             const CUtensorMap& mapC, const GemmArgs& a, int clusters,
                             cudaStream_t stream) {
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(gemm_pair_kernel), kMaxSmem);
  if (e != cudaSuccess) return e;
  if (a.mode == GEMM_HEAD || a.m_slabs % 2 != 0 || a.stages < 2 || a.pair || a.dense_pair ||
      gemm_pair_smem_bytes(a) > (size_t)kMaxSmem)
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = gemm_pair_smem_bytes(a);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, gemm_pair_kernel, mapA, mapB_half, mapC, a);
}

}  // namespace dg
