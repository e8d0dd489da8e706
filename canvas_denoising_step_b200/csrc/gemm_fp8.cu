// Expert GEMMs (GATEUP, DOWN) with FP8 E4M3 weights and bf16 activations on the
// bf16 tcgen05 MMA, for sm_100a.
//
// Each weight row r of a group g is stored as E4M3 codes q with one fp32 scale
// s[g][r]; the layer uses q * s.  The codes stream in at one byte per element
// into a deep ring of 64-element k-blocks; converter warps expand every
// [rows x 64] code tile into the bf16 K-major 128-byte-swizzle operand the MMA
// reads (E4M3 values are exact in bf16); the epilogue multiplies each weight
// row's accumulator by its scale.  Tiles are dealt longest chunk first from the
// router's order and a counter, as in the bf16 engine (gemm_tc.cu), and the
// epilogues are that engine's.
//
// Roles (352 threads):
//   warp 0, lane 0   takes each next tile from the counter and publishes it to
//                    the other roles (a 4-deep queue), then loads its code
//                    tiles (W ring, TMA)
//   warp 1           TMEM allocation; lane 0 issues the MMAs (A from the A ring,
//                    B from the B ring)
//   warps 2..5       epilogue
//   warps 6..9       converters (W ring -> A ring)
//   warp 10, lane 0  activation tiles (B ring, TMA); in DOWN it first waits for
//                    the gate/up epilogues of the tile's chunk (hand-over counters)
#include <cuda_fp8.h>

#include "gemm_shared.cuh"

namespace dg {

namespace {

constexpr int kFp8Threads = 352;
constexpr int kFp8MaxSmem = 232448;
constexpr int kWTileBytes = 128 * 64;   // 128 rows x 64 codes

// 16 E4M3 codes -> 16 bf16 (two 16-byte chunks), exactly, in integer and packed
// bf16 arithmetic (the conversion instructions run on a narrow pipe and could
// not keep up with the weight stream).  A code s.eeee.mmm placed as bf16 bits
// s.0000eeee.mmm0000 is the code's value times 2^-120 (e >= 1: (1 + m/8) 2^(e-127);
// e = 0: the bf16 subnormal m/8 2^-126 = m 2^-9 2^-120); one bf16x2 multiply by
// 2^120 restores it, exactly, since every E4M3 value is a normal bf16.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two) {
  // two: codes in bits [7:0] and [23:16]
  const uint32_t bits = ((two & 0x007F007Fu) << 4) | ((two & 0x00800080u) << 8);
  __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&bits);
  const __nv_bfloat162 k = __floats2bfloat162_rn(0x1p120f, 0x1p120f);
  v = __hmul2(v, k);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void e4m3x16_to_bf16(const uint4 c, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = e4m3x2_to_bf16x2(__byte_perm(w[i], 0u, 0x4140));      // codes 0, 1 of the word
    o[2 * i + 1] = e4m3x2_to_bf16x2(__byte_perm(w[i], 0u, 0x4342));  // codes 2, 3
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

}  // namespace

__global__ void __launch_bounds__(kFp8Threads, 1)
gemm_fp8_kernel(const __grid_constant__ CUtensorMap mapW, const __grid_constant__ CUtensorMap mapB,
                const __grid_constant__ CUtensorMap mapC, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int SW = a.stages;                       // W stages
  const int SA = a.sa, SB = a.sb;                // A (bf16) and B stages
  const int n_w = a.pair ? 2 : 1;                // 128-row code tiles per W / A stage
  const uint32_t w_stage = (uint32_t)(n_w * kWTileBytes);
  const uint32_t a_stage = (uint32_t)(n_w * kATileBytes);
  const uint32_t b_stage = (uint32_t)a.b_bytes;
  // layout: A ring | B ring | W ring | barriers (1 KB) | tables | output staging
  const uint32_t off_a = 0, off_b = SA * a_stage, off_w = off_b + SB * b_stage;
  const uint32_t off_bar = off_w + (uint32_t)SW * w_stage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + off_bar);
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_u32(bars);
  // barrier slots: w full/empty [SW], a full/empty [SA], b full/empty [SB],
  // tmem full/empty [2], tile queue full/empty [kTileQ]
  auto w_full = [&](int s) { return bar_base + 8u * s; };
  auto w_empty = [&](int s) { return bar_base + 8u * (SW + s); };
  auto a_full = [&](int s) { return bar_base + 8u * (2 * SW + s); };
  auto a_empty = [&](int s) { return bar_base + 8u * (2 * SW + SA + s); };
  auto b_full = [&](int s) { return bar_base + 8u * (2 * SW + 2 * SA + s); };
  auto b_empty = [&](int s) { return bar_base + 8u * (2 * SW + 2 * SA + SB + s); };
  const int tb0 = 2 * SW + 2 * SA + 2 * SB;
  auto tfull_bar = [&](int b) { return bar_base + 8u * (tb0 + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (tb0 + 2 + b); };
  auto tq_full_bar = [&](int q) { return bar_base + 8u * (tb0 + 4 + q); };
  auto tq_empty_bar = [&](int q) { return bar_base + 8u * (tb0 + 4 + kTileQ + q); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + tb0 + 4 + 2 * kTileQ);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_tq = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < SW; ++s) {
      mbar_init(w_full(s), 1);
      mbar_init(w_empty(s), 4);        // the four converter warps
    }
    for (int s = 0; s < SA; ++s) {
      mbar_init(a_full(s), 4);         // the four converter warps
      mbar_init(a_empty(s), 1);        // the MMA commit
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(b_full(s), 1);
      mbar_init(b_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 4);
    }
    for (int q = 0; q < kTileQ; ++q) {
      mbar_init(tq_full_bar(q), 1);
      mbar_init(tq_empty_bar(q), 10);  // MMA, 4 epilogue warps, 4 converter warps, B loader
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mapW);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // group tables and chunk order (written by the router, which has completed:
  // see the bf16 engine)
  int* s_prefix = reinterpret_cast<int*>(smem + off_bar + 1024);
  int* s_offsets = s_prefix + (a.n_groups + 1);
  int* s_order = a.chunk_order ? s_offsets + (a.n_groups + 1) : nullptr;
  float* s_stage_out = reinterpret_cast<float*>(smem + off_bar + 1024 + a.tab_bytes);
  for (int i = threadIdx.x; i <= a.n_groups; i += blockDim.x) {
    s_prefix[i] = __ldcg(a.chunk_prefix + i);
    s_offsets[i] = __ldcg(a.offsets + i);
  }
  __syncthreads();
  if (s_order)
    for (int i = threadIdx.x; i < s_prefix[a.n_groups]; i += blockDim.x)
      s_order[i] = __ldcg(a.chunk_order + i);
  __syncthreads();
  const int n_tiles = tile_count(a, s_prefix);

  // The first tile and its first code stages go out before the grid wait (the
  // weights do not depend on the previous kernel).
  int first_t = -1, pre = 0;
  if (warp == 0 && lane == 0) {
    first_t = atomicAdd(a.tile_counter, 1);
    if (first_t < n_tiles) {
      const TileInfo ti = decode_tile(a, first_t, s_prefix, s_offsets, s_order);
      pre = min(SW, ti.kb1 - ti.kb0);
      for (int p = 0; p < pre; ++p) {
        mbar_arrive_expect_tx(w_full(p), (uint32_t)(ti.n_acc * kWTileBytes));
        for (int i = 0; i < ti.n_acc; ++i)
          tma_load_3d(smem_base + off_w + (uint32_t)p * w_stage + (uint32_t)(i * kWTileBytes),
                      &mapW, w_full(p), (ti.kb0 + p) * kBK, ti.a_row0 + i * 128, ti.g);
      }
    }
  }
  const bool handover = a.mode == GEMM_DOWN && a.chunk_ready != nullptr;
  if (!handover) griddep_wait();
  griddep_launch();

  // consumers of the tile queue: returns the tile of iteration `it`, or -1 at the end
  auto next_tile = [&](int it, bool arrive_one) -> int {
    const int q = it % kTileQ;
    if (!mbar_wait(tq_full_bar(q), (uint32_t)((it / kTileQ) & 1), abort_flag, a.err)) return -2;
    const int t = s_tq[q];
    if (arrive_one) mbar_arrive(tq_empty_bar(q));
    return t;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ tile fetch + code loads
      int iw = 0;   // W stages issued
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int q = it % kTileQ;
        if (!mbar_wait(tq_empty_bar(q), (uint32_t)((it / kTileQ) & 1) ^ 1u, abort_flag, a.err)) {
          ok = false;
          break;
        }
        int t = it == 0 ? first_t : atomicAdd(a.tile_counter, 1);
        if (t >= n_tiles) t = -1;
        s_tq[q] = t;
        mbar_arrive(tq_full_bar(q));
        if (t < 0) break;
        const TileInfo ti = decode_tile(a, t, s_prefix, s_offsets, s_order);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++iw) {
          if (it == 0 && kb - ti.kb0 < pre) continue;   // issued before the grid wait
          const int s = iw % SW;
          if (!mbar_wait(w_empty(s), (uint32_t)((iw / SW) & 1) ^ 1u, abort_flag, a.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(w_full(s), (uint32_t)(ti.n_acc * kWTileBytes));
          for (int i = 0; i < ti.n_acc; ++i)
            tma_load_3d(smem_base + off_w + (uint32_t)s * w_stage + (uint32_t)(i * kWTileBytes),
                        &mapW, w_full(s), kb * kBK, ti.a_row0 + i * 128, ti.g);
        }
      }
      if (!ok)   // abort path: let the issued copies land
        for (int j = (iw > SW ? iw - SW : 0); j < iw; ++j)
          mbar_drain(w_full(j % SW), (uint32_t)((j / SW) & 1));
    }
    __syncwarp();
  } else if (warp == 10) {
    if (lane == 0) {
      // ------------------------------------------------ activation loads
      int ib = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int t = next_tile(it, true);
        if (t == -2) { ok = false; break; }
        if (t < 0) break;
        const TileInfo ti = decode_tile(a, t, s_prefix, s_offsets, s_order);
        if (handover) {
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
          fence_proxy_async_global();
        }
        const uint32_t tx = (uint32_t)(ti.n_bbox * a.b_box_rows * 128);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++ib) {
          const int s = ib % SB;
          if (!mbar_wait(b_empty(s), (uint32_t)((ib / SB) & 1) ^ 1u, abort_flag, a.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(b_full(s), tx);
          for (int i = 0; i < ti.n_bbox; ++i)
            tma_load_2d(smem_base + off_b + (uint32_t)s * b_stage + (uint32_t)(i * a.b_box_rows * 128),
                        &mapB, b_full(s), kb * kBK, ti.row0 + i * a.b_box_rows);
        }
      }
      if (!ok)
        for (int j = (ib > SB ? ib - SB : 0); j < ib; ++j)
          mbar_drain(b_full(j % SB), (uint32_t)((j / SB) & 1));
    }
    __syncwarp();
  } else if (warp >= 6) {
    // ------------------------------------------------ converters
    // thread c (0..127) takes, in each of four passes, 16 codes (one 16-byte
    // chunk) of row p * 32 + c / 4: a warp reads 8 whole 64-byte rows and writes
    // their 16 bf16 chunks into the 128-byte-swizzle layout (chunk k of row r at
    // k ^ (r % 8))
    const int c = threadIdx.x - 192;
    const int cq = c & 3;
    int iw = 0, ia = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int t = next_tile(it, false);
      __syncwarp();
      if (lane == 0 && t != -2) mbar_arrive(tq_empty_bar(it % kTileQ));
      if (t == -2) { ok = false; break; }
      if (t < 0) break;
      const TileInfo ti = decode_tile(a, t, s_prefix, s_offsets, s_order);
      for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++iw, ++ia) {
        const int sw = iw % SW, sa = ia % SA;
        if (!__all_sync(0xffffffffu, mbar_wait(w_full(sw), (uint32_t)((iw / SW) & 1), abort_flag, a.err)) ||
            !__all_sync(0xffffffffu, mbar_wait(a_empty(sa), (uint32_t)((ia / SA) & 1) ^ 1u, abort_flag, a.err))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* wsrc = smem + off_w + (uint32_t)sw * w_stage;
        const uint32_t adst = smem_base + off_a + (uint32_t)sa * a_stage;
        for (int i = 0; i < ti.n_acc; ++i) {
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const int row = p * 32 + (c >> 2);
            const uint4 codes = *reinterpret_cast<const uint4*>(wsrc + i * kWTileBytes + row * 64 + cq * 16);
            uint4 lo, hi;
            e4m3x16_to_bf16(codes, lo, hi);
            const uint32_t rbase = adst + (uint32_t)(i * kATileBytes + row * 128);
            st_shared_v4(rbase + (uint32_t)(((2 * cq) ^ (row & 7)) * 16), lo.x, lo.y, lo.z, lo.w);
            st_shared_v4(rbase + (uint32_t)(((2 * cq + 1) ^ (row & 7)) * 16), hi.x, hi.y, hi.z, hi.w);
          }
        }
        fence_proxy_async_smem();   // the MMA (async proxy) reads what this thread wrote
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(w_empty(sw));
          mbar_arrive(a_full(sa));
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const int n_bufs = a.n_bufs;
      const uint32_t buf_cols = 512u / (uint32_t)n_bufs;
      int ia = 0, ib = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int t = next_tile(it, true);
        if (t == -2 || t < 0) break;
        const TileInfo ti = decode_tile(a, t, s_prefix, s_offsets, s_order);
        const int buf = it % n_bufs;
        if (!mbar_wait(tempty_bar(buf), (uint32_t)((it / n_bufs) & 1) ^ 1u, abort_flag, a.err)) break;
        tc_fence_after();
        const uint32_t d_base = tmem_base + (uint32_t)buf * buf_cols;
        const uint32_t idesc = idesc_bf16_f32(ti.n_mma);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++ia, ++ib) {
          const int sa = ia % SA, sb = ib % SB;
          if (!mbar_wait(a_full(sa), (uint32_t)((ia / SA) & 1), abort_flag, a.err) ||
              !mbar_wait(b_full(sb), (uint32_t)((ib / SB) & 1), abort_flag, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_base + off_a + (uint32_t)sa * a_stage;
          const uint32_t sB = smem_base + off_b + (uint32_t)sb * b_stage;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bdesc = sdesc_kmajor_sw128(sB + kk * 32);
            for (int i = 0; i < ti.n_acc; ++i)
              umma_bf16(d_base + (uint32_t)i * kAccCols, sdesc_kmajor_sw128(sA + i * kATileBytes + kk * 32),
                        bdesc, idesc, (kb > ti.kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(a_empty(sa));
          umma_commit(b_empty(sb));
        }
        if (!ok) break;
        umma_commit(tfull_bar(buf));
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;
    const int n_bufs = a.n_bufs;
    const uint32_t buf_cols = 512u / (uint32_t)n_bufs;
    const int n_sbuf = a.epi_bytes / (4 * 4096);
    float* s_warp_out = s_stage_out + (warp - 2) * n_sbuf * 1024;
    int sbuf = 0;
    for (int it = 0;; ++it) {
      const int t = next_tile(it, false);
      __syncwarp();
      if (lane == 0 && t != -2) mbar_arrive(tq_empty_bar(it % kTileQ));
      if (t < 0) break;
      const TileInfo ti = decode_tile(a, t, s_prefix, s_offsets, s_order);
      const int buf = it % n_bufs;
      if (!mbar_wait(tfull_bar(buf), (uint32_t)((it / n_bufs) & 1), abort_flag, a.err)) break;
      tc_fence_after();
      const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)buf * buf_cols;
      if (a.mode == GEMM_DOWN)
        epi_f32_tile(a, &mapC, ti, lane_addr, q, lane, s_warp_out, n_sbuf, sbuf, a.w_scale);
      else
        epi_gateup_tile(a, &mapC, ti, lane_addr, q, lane,
                        smem_u32(s_stage_out) + (uint32_t)(warp - 2) * 2048u, sbuf, a.w_scale);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(buf));
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ============================================================================ host side

// Shared-memory plan of the FP8-weight GEMM: A (bf16, 2 stages) and B (3
// stages) rings, as many W (code) stages as fit beside the barriers, tables and
// output staging, at most 16.
void gemm_fp8_plan_smem(GemmArgs& a) {
  const int n_w = a.pair ? 2 : 1;
  a.sa = 2;
  a.sb = 3;
  const int SA = a.sa, SB = a.sb;
  a.n_bufs = n_w == 1 ? 2 : 1;
  a.tab_bytes = ((2 * (a.n_groups + 1) * 4 + (a.chunk_order ? a.max_chunks * 4 : 0) + 127) / 128) * 128;
  a.epi_bytes = a.mode == GEMM_DOWN ? 4 * 4096 : 2 * 4 * 1024;
  a.a_bytes = n_w * kATileBytes;
  if (a.b_box_rows <= 0) a.b_box_rows = 32;
  a.b_bytes = ((a.n_tile + a.b_box_rows - 1) / a.b_box_rows) * a.b_box_rows * 128;
  const int fixed = 1024 + SA * a.a_bytes + SB * a.b_bytes + 1024 + a.tab_bytes + a.epi_bytes;
  int s = (kFp8MaxSmem - fixed) / (n_w * kWTileBytes);
  a.stages = s > 16 ? 16 : s;
  a.stage_bytes = n_w * kWTileBytes;
}

size_t gemm_fp8_smem_bytes(const GemmArgs& a) {
  return 1024 + (size_t)a.sa * a.a_bytes + (size_t)a.sb * a.b_bytes + (size_t)a.stages * a.stage_bytes +
         1024 + a.tab_bytes + a.epi_bytes;
}

cudaError_t gemm_fp8_launch(const CUtensorMap& mapW, const CUtensorMap& mapB, const CUtensorMap& mapC,
                            const GemmArgs& a, int grid, cudaStream_t stream) {
  if ((a.mode != GEMM_GATEUP && a.mode != GEMM_DOWN) || !a.tile_counter || !a.w_scale ||
      a.pair || a.stages < 4)
    return cudaErrorInvalidValue;
  if (gemm_fp8_smem_bytes(a) > (size_t)kFp8MaxSmem) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(gemm_fp8_kernel), kFp8MaxSmem);
  if (e != cudaSuccess) return e;
  return launch_k(gemm_fp8_kernel, dim3(grid), dim3(kFp8Threads), gemm_fp8_smem_bytes(a), stream,
                  mapW, mapB, mapC, a);
}

// bf16 [rows][K] -> E4M3 codes [rows][K] and fp32 scales [rows]: one warp per row,
// s = max|w| / 448 (fp32 division), q = E4M3(w / s) round to nearest even.
__global__ void quantize_rows_kernel(const bf16* src, uint8_t* dst, float* scale, long long rows,
                                     int K) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const bf16* w = src + row * K;
  float amax = 0.f;
  for (int k = lane; k < K; k += 32) amax = fmaxf(amax, fabsf(bf16_to_f(w[k])));
  amax = warp_max(amax);
  const float s = __fdiv_rn(amax, 448.0f);
  if (lane == 0) scale[row] = s;
  uint8_t* q = dst + row * K;
  for (int k = lane; k < K; k += 32)
    q[k] = s > 0.f ? (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(bf16_to_f(w[k]), s), __NV_SATFINITE, __NV_E4M3)
                   : (uint8_t)0;
}

cudaError_t launch_quantize_rows(const bf16* src, uint8_t* dst, float* scale, long long rows, int K,
                                 cudaStream_t s) {
  const int warps = 8;
  quantize_rows_kernel<<<(unsigned)((rows + warps - 1) / warps), 32 * warps, 0, s>>>(src, dst, scale,
                                                                                   rows, K);
  return cudaGetLastError();
}

}  // namespace dg
