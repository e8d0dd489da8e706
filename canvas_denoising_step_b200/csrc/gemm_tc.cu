// Persistent, warp-specialised tcgen05 GEMM for sm_100a.
//
// Roles (192 threads): warp 0 lane 0 issues TMA loads into a ring of shared
// memory stages; warp 1 lane 0 issues tcgen05.mma into TMEM accumulators
// (warp 1 also allocates TMEM); warps 2..5 are the epilogue, each reading its
// 32-lane quadrant of TMEM with tcgen05.ld.  Accumulators are double
// buffered so the epilogue of one tile overlaps the MMAs of the next.
// The fp32 outputs (DENSE, DOWN) leave through shared memory: each epilogue
// warp stages a 32 x 32 block and one lane writes it with a TMA tensor store
// (blocks that end inside a group's rows, in DOWN, are written with masked
// 16-byte stores instead, so that no row of the next group is touched).
// The grouped modes copy the group tables (chunk prefix, row offsets) into
// shared memory once, so tile decoding does not walk global memory.
//
// Operands are K-major bf16 tiles with the 128-byte swizzle (64 elements of
// K per row).  The MMA is always M = 128: "A" rows are the output features
// for the weight-streaming modes (the weight is the M operand, the few
// activation rows are N), and the token rows for the vocab head.
//
// Modes
//  DENSE   Y[s][n][m] = sum_{k in split s} X[n][k] W[m][k]      (fp32 split-K partials);
//          with dense_pair a tile holds two 128-row weight slabs sharing one B tile
//  GATEUP  H[r][f] = silu(g) * u, with g/u the gate/up rows 2f/2f+1 of the
//          group's interleaved weight, for rows r of the group     (bf16)
//  DOWN    Y[r][m] = sum_k H[r][k] Wd[g][m][k]                   (fp32)
//  HEAD    per token row t and 256-wide vocab block b: the max logit, its
//          index (lowest on ties) and sum exp(l - max) over the block, with
//          the mask id and out-of-range vocab rows excluded      (partials);
//          with inv_temp set, the sums are taken of exp(z) and z exp(z) with
//          z = (l - max) * inv_temp (the entropy of the block at that temperature)
#include "gemm_shared.cuh"

namespace dg {

namespace {

constexpr int kThreads = 192;
}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
               const __grid_constant__ CUtensorMap mapC, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int S = a.stages;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)S * a.stage_bytes);
  // full[0..S), empty[S..2S), tmem_full[2S..2S+2), tmem_empty[2S+2..2S+4),
  // tile queue full / empty [2S+4 .. 2S+4+2*kTileQ)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4 + 2 * kTileQ);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_tq = reinterpret_cast<volatile int*>(tmem_slot + 2);   // [kTileQ] tiles
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_u32(bars);
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (S + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * S + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * S + 2 + b); };
  auto tq_full_bar = [&](int q) { return bar_base + 8u * (2 * S + 4 + q); };
  auto tq_empty_bar = [&](int q) { return bar_base + 8u * (2 * S + 4 + kTileQ + q); };
  // grouped modes with a tile counter deal tiles dynamically: the producer takes
  // the next tile from the counter and passes it to the MMA and epilogue warps
  // through a small queue; otherwise CTA b takes tiles b, b + grid, ...
  const bool dyn = (a.mode == GEMM_GATEUP || a.mode == GEMM_DOWN) && a.tile_counter != nullptr;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 4);
    }
    for (int q = 0; q < kTileQ; ++q) {
      mbar_init(tq_full_bar(q), 1);
      mbar_init(tq_empty_bar(q), 5);   // the MMA lane and the four epilogue warps
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mapA);
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
  // Everything above overlaps the previous kernel's tail.
  //
  // The group tables of the grouped modes come from the router, two or three
  // kernels back.  The router, the row gather and the gate/up GEMM each call
  // griddepcontrol.launch_dependents only after their own grid wait, so the
  // router had completed before the kernel just before this one let it
  // launch: the tables are read before this kernel's wait.
  int* s_prefix = reinterpret_cast<int*>(smem + (size_t)S * a.stage_bytes + 1024);
  int* s_offsets = s_prefix + (a.n_groups + 1);
  int* s_order = a.chunk_order ? s_offsets + (a.n_groups + 1) : nullptr;
  float* s_stage_out = reinterpret_cast<float*>(smem + (size_t)S * a.stage_bytes + 1024 + a.tab_bytes);
  const bool grouped = a.mode == GEMM_GATEUP || a.mode == GEMM_DOWN;
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
  // The weights do not depend on the previous kernel either: the producer
  // issues the weight operand of its first tile's first stages now (fresh
  // barriers, no empty waits), and the activation operand after the wait.
  int pre = 0;
  int first_t = blockIdx.x;
  // the first dynamic tile (the counter was zeroed by the router, which has
  // completed, as the tables above)
  if (dyn && warp == 0 && lane == 0) first_t = atomicAdd(a.tile_counter, 1);
  if (warp == 0 && lane == 0 && first_t < tile_count(a, s_prefix)) {
    const TileInfo ti = decode_tile(a, first_t, s_prefix, s_offsets, s_order);
    const uint32_t tx = (uint32_t)(ti.n_acc * kATileBytes) +
                        (uint32_t)(ti.n_bbox * a.b_box_rows * 128);
    pre = min(S, ti.kb1 - ti.kb0);
    for (int p = 0; p < pre; ++p) {
      const uint32_t sA = smem_base + (uint32_t)p * a.stage_bytes;
      const int kx = (ti.kb0 + p) * kBK;
      mbar_arrive_expect_tx(full_bar(p), tx);
      if (a.mode == GEMM_DENSE) {
        for (int i = 0; i < ti.n_acc; ++i)
          tma_load_2d(sA + i * kATileBytes, &mapA, full_bar(p), kx, ti.a_row0 + i * 128);
      } else if (a.mode == GEMM_HEAD) {
        tma_load_2d(sA + (uint32_t)a.a_bytes, &mapB, full_bar(p), kx, ti.row0);
      } else {
        for (int i = 0; i < ti.n_acc; ++i)
          tma_load_3d(sA + i * kATileBytes, &mapA, full_bar(p), kx, ti.a_row0 + i * 128, ti.g);
      }
    }
  }
  // Data written by the previous kernel is read from here on.  A DOWN launch
  // with ready counters does not wait for the whole gate/up grid: its H rows
  // are guarded per chunk below.
  const bool handover = a.mode == GEMM_DOWN && a.chunk_ready != nullptr;
  if (!handover) griddep_wait();
  griddep_launch();

  const int n_tiles = tile_count(a, s_prefix);
  // TMEM layout: n_bufs tile buffers of 512/n_bufs columns; in a buffer,
  // accumulator i starts at column i * kAccCols.
  const int n_bufs = a.n_bufs;
  const uint32_t buf_cols = 512u / (uint32_t)n_bufs;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      bool wrapped = false, ok = true;
      for (int it = 0; ok; ++it) {
        int t;
        if (dyn) {
          // take the next tile and publish it to the MMA and epilogue warps
          const int q = it % kTileQ;
          if (!mbar_wait(tq_empty_bar(q), (uint32_t)((it / kTileQ) & 1) ^ 1u, abort_flag, a.err)) {
            ok = false;
            break;
          }
          t = it == 0 ? first_t : atomicAdd(a.tile_counter, 1);
          if (t >= n_tiles) t = -1;
          s_tq[q] = t;
          mbar_arrive(tq_full_bar(q));
          if (t < 0) break;
        } else {
          t = blockIdx.x + it * gridDim.x;
          if (t >= n_tiles) break;
        }
        const bool first = it == 0;
        const TileInfo ti = decode_tile(a, t, s_prefix, s_offsets, s_order);
        const uint32_t tx = (uint32_t)(ti.n_acc * kATileBytes) +
                            (uint32_t)(ti.n_bbox * a.b_box_rows * 128);
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
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          // the weight operand of this stage went out before the grid wait
          const bool weight_issued = first && kb - ti.kb0 < pre;
          const uint32_t sA = smem_base + (uint32_t)stage * a.stage_bytes;
          const uint32_t sB = sA + (uint32_t)a.a_bytes;
          const uint32_t fb = full_bar(stage);
          const int kx = kb * kBK;
          if (!weight_issued) {
            if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.err)) { ok = false; break; }
            mbar_arrive_expect_tx(fb, tx);
          }
          if (a.mode == GEMM_DENSE) {
            if (!weight_issued)
              for (int i = 0; i < ti.n_acc; ++i)
                tma_load_2d(sA + i * kATileBytes, &mapA, fb, kx, ti.a_row0 + i * 128);
          } else if (a.mode == GEMM_HEAD) {
            for (int i = 0; i < ti.n_acc; ++i)
              tma_load_2d(sA + i * kATileBytes, &mapA, fb, kx, ti.a_row0 + i * 128);
          } else if (!weight_issued) {
            for (int i = 0; i < ti.n_acc; ++i)
              tma_load_3d(sA + i * kATileBytes, &mapA, fb, kx, ti.a_row0 + i * 128, ti.g);
          }
          if (!(weight_issued && a.mode == GEMM_HEAD))
            for (int i = 0; i < ti.n_bbox; ++i)
              tma_load_2d(sB + (uint32_t)(i * a.b_box_rows * 128), &mapB, fb, kx,
                          ti.row0 + i * a.b_box_rows);
          if (++stage == S) { stage = 0; phase ^= 1u; wrapped = true; }
        }
      }
      if (!ok) {  // abort path: let issued copies land before the CTA exits
        for (int s = 0; s < S; ++s) {
          if (s < stage) mbar_drain(full_bar(s), phase);
          else if (wrapped) mbar_drain(full_bar(s), phase ^ 1u);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        int t;
        if (dyn) {
          const int q = it % kTileQ;
          if (!mbar_wait(tq_full_bar(q), (uint32_t)((it / kTileQ) & 1), abort_flag, a.err)) break;
          t = s_tq[q];
          mbar_arrive(tq_empty_bar(q));
          if (t < 0) break;
        } else {
          t = blockIdx.x + it * gridDim.x;
          if (t >= n_tiles) break;
        }
        const TileInfo ti = decode_tile(a, t, s_prefix, s_offsets, s_order);
        const int buf = it % n_bufs;
        const uint32_t tph = (uint32_t)((it / n_bufs) & 1);
        if (!mbar_wait(tempty_bar(buf), tph ^ 1u, abort_flag, a.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_base = tmem_base + (uint32_t)buf * buf_cols;
        const uint32_t idesc = idesc_bf16_f32(ti.n_mma);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sA = smem_base + (uint32_t)stage * a.stage_bytes;
          const uint32_t sB = sA + (uint32_t)a.a_bytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bdesc = sdesc_kmajor_sw128(sB + kk * 32);
            for (int i = 0; i < ti.n_acc; ++i) {
              const uint64_t adesc = sdesc_kmajor_sw128(sA + i * kATileBytes + kk * 32);
              umma_bf16(d_base + (uint32_t)i * kAccCols, adesc, bdesc, idesc,
                        (kb > ti.kb0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(empty_bar(stage));
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(tfull_bar(buf));
      }
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;            // accumulator row (TMEM lane)
    // staging blocks of this warp for the fp32 outputs: n_sbuf of 32 x 32 fp32
    const int n_sbuf = a.epi_bytes / (4 * 4096);
    float* s_warp_out = s_stage_out + (warp - 2) * n_sbuf * 1024;
    int sbuf = 0;
    for (int it = 0;; ++it) {
      int t;
      if (dyn) {
        const int q = it % kTileQ;
        if (!mbar_wait(tq_full_bar(q), (uint32_t)((it / kTileQ) & 1), abort_flag, a.err)) break;
        t = s_tq[q];
        __syncwarp();
        if (lane == 0) mbar_arrive(tq_empty_bar(q));
        if (t < 0) break;
      } else {
        t = blockIdx.x + it * gridDim.x;
        if (t >= n_tiles) break;
      }
      const TileInfo ti = decode_tile(a, t, s_prefix, s_offsets, s_order);
      const int buf = it % n_bufs;
      const uint32_t tph = (uint32_t)((it / n_bufs) & 1);
      if (!mbar_wait(tfull_bar(buf), tph, abort_flag, a.err)) break;
      tc_fence_after();
      const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)buf * buf_cols;
      uint32_t v[32];
      if (a.mode == GEMM_DENSE || a.mode == GEMM_DOWN) {
        epi_f32_tile(a, &mapC, ti, lane_addr, q, lane, s_warp_out, n_sbuf, sbuf, nullptr);
      } else if (a.mode == GEMM_GATEUP) {
        epi_gateup_tile(a, &mapC, ti, lane_addr, q, lane,
                        smem_u32(s_stage_out) + (uint32_t)(warp - 2) * 2048u, sbuf, nullptr);
      } else if (a.inv_temp == nullptr) {  // HEAD
        for (int i = 0; i < ti.n_acc; ++i) {
          const int tok_row = ti.tb * 256 + i * 128 + r;
          float mx = -INFINITY, sum = 0.f;
          int arg = -1;
          for (int c0 = 0; c0 < 256; c0 += 32) {
            tmem_ld32(lane_addr + (uint32_t)i * kAccCols + (uint32_t)c0, v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int vid = ti.row0 + c0 + j;
              if (vid < a.vocab && vid != a.mask_id) {
                const float x = __uint_as_float(v[j]);
                if (x > mx) {
                  sum = sum * __expf(mx - x) + 1.0f;
                  mx = x;
                  arg = vid;
                } else {
                  sum += __expf(x - mx);
                }
              }
            }
          }
          if (tok_row < a.T) {
            const size_t o = (size_t)ti.vb * a.T + tok_row;
            a.head_m[o] = mx;
            a.head_s[o] = sum;
            a.head_a[o] = arg;
          }
        }
      } else {  // HEAD with the entropy statistics at temperature 1 / inv_temp
        // z = (l - mx) / temp; S = sum e^z; Q = sum z e^z; when the max grows by
        // d = (mx_old - mx_new) / temp, S <- e^d S and Q <- e^d (Q + d S).
        const float it = *a.inv_temp;
        for (int i = 0; i < ti.n_acc; ++i) {
          const int tok_row = ti.tb * 256 + i * 128 + r;
          float mx = -INFINITY, sum = 0.f, qz = 0.f;
          int arg = -1;
          for (int c0 = 0; c0 < 256; c0 += 32) {
            tmem_ld32(lane_addr + (uint32_t)i * kAccCols + (uint32_t)c0, v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int vid = ti.row0 + c0 + j;
              if (vid < a.vocab && vid != a.mask_id) {
                const float x = __uint_as_float(v[j]);
                if (x > mx) {
                  if (arg < 0) {
                    sum = 1.0f;
                    qz = 0.f;
                  } else {
                    const float dz = (mx - x) * it;
                    const float e = __expf(dz);
                    qz = e * (qz + dz * sum);
                    sum = e * sum + 1.0f;
                  }
                  mx = x;
                  arg = vid;
                } else {
                  const float z = (x - mx) * it;
                  const float e = __expf(z);
                  sum += e;
                  qz += z * e;
                }
              }
            }
          }
          if (tok_row < a.T) {
            const size_t o = (size_t)ti.vb * a.T + tok_row;
            a.head_m[o] = mx;
            a.head_s[o] = sum;
            a.head_a[o] = arg;
            a.head_q[o] = qz;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(buf));
    }
    // tensor stores of this warp complete before the CTA exits
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

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

bool make_tmap_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                  uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid,
                  uint64_t outer, uint32_t box_mid) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {inner * 2, inner * mid * 2};
  cuuint32_t box[3] = {64, box_mid, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 8-bit codes [outer][mid][inner] read in boxes of 64 codes x 128 rows (no swizzle:
// a box lands as 128 rows of 64 bytes).
bool make_tmap_3d_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid,
                     uint64_t outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {inner, inner * mid};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 output [outer][mid][inner] written in 32 x 32 blocks (no swizzle):
// elements past any extent are not written by a tensor store.
bool make_tmap_out_f32(CUtensorMap* map, float* base, uint64_t inner, uint64_t mid,
                       uint64_t outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {inner * 4, inner * mid * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [outer][inner] written in [32 rows][16] blocks (the gate/up H stores).
bool make_tmap_h_store(CUtensorMap* map, void* base, uint64_t inner, uint64_t outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {16, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 [outer][inner] written in 32 x 32 blocks whose shared-memory image has
// the 128-byte swizzle (16-byte chunk c of row r at chunk c ^ (r % 8)).
bool make_tmap_f32_sw128(CUtensorMap* map, float* base, uint64_t inner, uint64_t outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Shared-memory plan: A region (1 or 2 tiles of 16 KB) + B region, as many
// stages as fit beside the barriers, group tables and output staging; and the
// TMEM plan: two tile buffers of 256
// columns when a tile has one accumulator (so the epilogue of one tile
// overlaps the MMAs of the next), one buffer of two when it has two.
void gemm_plan_smem(GemmArgs& a) {
  const bool grouped = a.mode == GEMM_GATEUP || a.mode == GEMM_DOWN;
  const int n_a = (a.mode == GEMM_HEAD || (a.mode == GEMM_DENSE && a.dense_pair) ||
                   (grouped && a.pair)) ? 2 : 1;
  a.n_bufs = n_a == 1 ? 2 : 1;
  // group tables; fp32 output staging: two 4 KB blocks per epilogue warp for
  // DENSE, one for DOWN (which keeps its sixth operand stage)
  a.tab_bytes = grouped ? ((2 * (a.n_groups + 1) * 4 + (a.chunk_order ? a.max_chunks * 4 : 0) +
                            127) / 128) * 128 : 0;
  a.epi_bytes = a.mode == GEMM_DENSE ? 2 * 4 * 4096
                : (a.mode == GEMM_DOWN ? 4 * 4096 : (a.mode == GEMM_GATEUP ? 2 * 4 * 1024 : 0));
  a.a_bytes = n_a * kATileBytes;
  if (a.mode == GEMM_HEAD) {
    a.b_box_rows = 256;
    a.b_bytes = 256 * 128;
  } else {
    if (a.b_box_rows <= 0) a.b_box_rows = 32;   // must match the B tensor map's box
    a.b_bytes = ((a.n_tile + a.b_box_rows - 1) / a.b_box_rows) * a.b_box_rows * 128;
  }
  a.stage_bytes = a.a_bytes + a.b_bytes;  // multiples of 1024
  int s = (int)((kMaxSmem - 2048 - a.tab_bytes - a.epi_bytes) / a.stage_bytes);
  a.stages = s < 2 ? 2 : (s > 8 ? 8 : s);
}

size_t gemm_smem_bytes(const GemmArgs& a) {
  // alignment slack, stages, barriers (1 KB), group tables, output staging
  return 1024 + (size_t)a.stages * a.stage_bytes + 1024 + a.tab_bytes + a.epi_bytes;
}

cudaError_t gemm_tc_launch(const CUtensorMap& mapA, const CUtensorMap& mapB,
                           const CUtensorMap& mapC, const GemmArgs& a, int grid,
                           cudaStream_t stream) {
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(gemm_tc_kernel), kMaxSmem);
  if (e != cudaSuccess) return e;
  if (gemm_smem_bytes(a) > (size_t)kMaxSmem) return cudaErrorInvalidValue;
  return launch_k(gemm_tc_kernel, dim3(grid), dim3(kThreads), gemm_smem_bytes(a), stream, mapA,
                  mapB, mapC, a);
}

}  // namespace dg
