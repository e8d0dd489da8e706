// Tile decoding and tile epilogues shared by the sm_100a GEMM kernels (the bf16
// engine of gemm_tc.cu and the FP8-weight expert GEMMs of gemm_fp8.cu).
#pragma once

#include "dg_kernels.h"

namespace dg {

constexpr int kBK = 64;             // K elements per stage (128-byte rows)
constexpr int kATileBytes = 128 * 128;  // 128 rows x 128 B
constexpr uint32_t kAccCols = 256;      // TMEM columns between the accumulators of a tile
constexpr int kMaxSmem = 232448;        // dynamic shared memory per CTA (227 KB)

struct TileInfo {
  int g, m_slab, row0, rows, kb0, kb1, split, tb, vb;
  int chunk;   // grouped: the chunk (group-major numbering shared by GATEUP and DOWN)
  int a_row0;  // first A row of the tile (accumulator i covers a_row0 + 128 i ..)
  int n_acc;   // accumulators (A tiles) per tile
  int n_mma;   // MMA N
  int n_bbox;  // B boxes per stage
};

__device__ __forceinline__ int upper_bound_prefix(const int* prefix, int n, int c) {
  // largest g in [0, n) with prefix[g] <= c
  int lo = 0, hi = n;  // prefix[0] == 0 <= c
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (prefix[mid] <= c) lo = mid; else hi = mid;
  }
  return lo;
}

// s_prefix / s_offsets: the group tables in shared memory (grouped modes)
__device__ __forceinline__ int tile_count(const GemmArgs& a, const int* s_prefix) {
  switch (a.mode) {
    case GEMM_DENSE: return a.m_slabs * ((a.N + a.n_tile - 1) / a.n_tile) * a.k_splits;
    case GEMM_GATEUP:
    case GEMM_DOWN: return s_prefix[a.n_groups] * a.m_slabs;
    default: return a.n_vblocks * a.n_tblocks;
  }
}

// s_order: the chunks longest first (grouped modes with a chunk order), else NULL
__device__ __forceinline__ TileInfo decode_tile(const GemmArgs& a, int t, const int* s_prefix,
                                               const int* s_offsets, const int* s_order) {
  TileInfo ti;
  ti.g = 0; ti.split = 0; ti.tb = 0; ti.vb = 0; ti.n_acc = 1; ti.chunk = 0;
  if (a.mode == GEMM_DENSE) {
    const int n_chunks = (a.N + a.n_tile - 1) / a.n_tile;
    ti.m_slab = t % a.m_slabs;
    const int rest = t / a.m_slabs;
    const int chunk = rest % n_chunks;
    ti.split = rest / n_chunks;
    ti.row0 = chunk * a.n_tile;
    ti.rows = min(a.n_tile, a.N - ti.row0);
    ti.kb0 = (int)(((long long)ti.split * a.n_kb) / a.k_splits);
    ti.kb1 = (int)(((long long)(ti.split + 1) * a.n_kb) / a.k_splits);
    ti.n_acc = a.dense_pair ? 2 : 1;
    ti.a_row0 = ti.m_slab * 128 * ti.n_acc;
  } else if (a.mode == GEMM_GATEUP || a.mode == GEMM_DOWN) {
    // tile t = (k-th chunk of the order, weight slab): all slabs of the longest
    // chunk are dealt first; with `pair` a slab is 256 weight rows (two accumulators)
    ti.m_slab = t % a.m_slabs;
    const int k = t / a.m_slabs;
    const int c = s_order ? s_order[k] : k;
    ti.chunk = c;
    ti.g = upper_bound_prefix(s_prefix, a.n_groups, c);
    const int j = c - s_prefix[ti.g];
    const int beg = s_offsets[ti.g], end = s_offsets[ti.g + 1];
    ti.row0 = beg + j * a.n_tile;
    ti.rows = min(a.n_tile, end - ti.row0);
    ti.kb0 = 0;
    ti.kb1 = a.n_kb;
    ti.a_row0 = ti.m_slab * 128 * (a.pair ? 2 : 1);
    ti.n_acc = (a.pair && ti.a_row0 + 128 < a.M) ? 2 : 1;
  } else {  // HEAD
    ti.tb = t % a.n_tblocks;
    ti.vb = t / a.n_tblocks;
    ti.m_slab = 0;
    ti.row0 = ti.vb * 256;
    ti.rows = 256;
    ti.n_acc = (a.T - ti.tb * 256 > 128) ? 2 : 1;
    ti.kb0 = 0;
    ti.kb1 = a.n_kb;
    ti.a_row0 = ti.tb * 256;
  }
  if (a.mode == GEMM_HEAD) {
    ti.n_mma = 256;
    ti.n_bbox = 1;
  } else {
    ti.n_mma = (ti.rows + 15) & ~15;
    ti.n_bbox = (ti.rows + a.b_box_rows - 1) / a.b_box_rows;
  }
  return ti;
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

constexpr int kTileQ = 4;   // depth of the dynamic tile queue (grouped modes)

// DENSE / DOWN tile epilogue of one epilogue warp: its 32 TMEM lanes (weight
// rows m0 .. m0+31 of each accumulator) leave as fp32 out[split][row][m] through
// 32 x 32 shared-memory blocks and TMA tensor stores; a block that ends inside
// a group's rows (DOWN) is written with masked 16-byte stores instead.  With
// row_scale, each weight row's values are first multiplied by its scale
// (row_scale[g * M + m]).
__device__ __forceinline__ void epi_f32_tile(const GemmArgs& a, const CUtensorMap* mapC,
                                             const TileInfo& ti, uint32_t lane_addr, int q,
                                             int lane, float* s_warp_out, int n_sbuf, int& sbuf,
                                             const float* row_scale) {
  uint32_t v[32];
  // out[split][row][m]; this warp holds rows m0 .. m0+31 of the tile
  float* out = a.out_f32 + (size_t)ti.split * a.N * a.M;
  for (int i = 0; i < ti.n_acc; ++i) {
    const int m0 = ti.a_row0 + i * 128 + q * 32;
    for (int c0 = 0; c0 < ti.n_mma; c0 += 32) {
      tmem_ld32(lane_addr + (uint32_t)i * kAccCols + (uint32_t)c0, v);
      tmem_wait_ld();
      if (row_scale && m0 + lane < a.M) {   // this lane's accumulator row is weight row m0 + lane
        const float sr = row_scale[(size_t)ti.g * a.M + m0 + lane];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * sr);
      }
      float* st = s_warp_out + sbuf * 1024;   // [32 rows n][32 m]
      // the store that last read this block has finished reading it
      if (lane == 0) {
        if (n_sbuf > 1) bulk_wait_read<1>(); else bulk_wait_read<0>();
      }
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 32; ++j) st[j * 32 + lane] = __uint_as_float(v[j]);
      if (a.mode == GEMM_DENSE || c0 + 32 <= ti.rows) {
        // rows past N (DENSE) and m past M are clipped by the tensor map;
        // a block with nothing inside is not stored at all
        if (m0 < a.M) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(mapC, smem_u32(st), m0, ti.row0 + c0, ti.split);
            bulk_commit();
          }
          sbuf = (sbuf + 1 == n_sbuf) ? 0 : sbuf + 1;
        }
      } else {
        __syncwarp();
#pragma unroll
        for (int it2 = 0; it2 < 8; ++it2) {
          const int nl = it2 * 4 + (lane >> 3), mo = 4 * (lane & 7);
          if (c0 + nl < ti.rows && m0 + mo < a.M)
            *reinterpret_cast<float4*>(out + (size_t)(ti.row0 + c0 + nl) * a.M + m0 + mo) =
                *reinterpret_cast<const float4*>(st + nl * 32 + mo);
        }
        __syncwarp();
      }
    }
  }
}

// GATEUP tile epilogue of one epilogue warp (one or two 128-row slabs per tile).  With
// row_scale, each interleaved gate / up row is first multiplied by its scale.
__device__ __forceinline__ void epi_gateup_tile(const GemmArgs& a, const CUtensorMap* mapC,
                                                const TileInfo& ti, uint32_t lane_addr, int q,
                                                int lane, uint32_t h_stage, int& sbuf,
                                                const float* row_scale) {
  uint32_t v[32];
  const int r = q * 32 + lane;
  for (int acc = 0; acc < ti.n_acc; ++acc) {   // accumulator acc: weight rows a_row0 + 128 acc ..
    const int row0 = ti.a_row0 + acc * 128;
    const float sr = row_scale ? row_scale[(size_t)ti.g * a.M + row0 + r] : 1.0f;
    // Interleaved rows: even accumulator rows are gate rows, odd rows the
    // matching up rows of the same output feature f.
    // A warp's 16 gate rows are 16 consecutive features f0 .. f0+15; a full
    // 32-row chunk of H leaves as one [32 rows][16 f] bf16 block through
    // shared memory and a tensor store (lanes 4p pack f0+2p, f0+2p+1);
    // a chunk that ends inside the group's rows is stored element-wise.
    const int f = (row0 + r) >> 1;
    const int f0 = (row0 + q * 32) >> 1;
    const bool is_gate = (r & 1) == 0;
    for (int c0 = 0; c0 < ti.n_mma; c0 += 32) {
      tmem_ld32(lane_addr + (uint32_t)acc * kAccCols + (uint32_t)c0, v);
      tmem_wait_ld();
      if (row_scale) {   // gate and up rows carry their own scales
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * sr);
      }
      if (c0 + 32 <= ti.rows && f0 + 16 <= a.F) {
        const uint32_t st = h_stage + (uint32_t)sbuf * 1024u;
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float x = __uint_as_float(v[j]);
          const float u = __shfl_xor_sync(0xffffffffu, x, 1);
          const float h = x / (1.0f + __expf(-x)) * u;       // meaningful in gate lanes
          const float h1 = __shfl_down_sync(0xffffffffu, h, 2);  // feature f + 1
          if ((lane & 3) == 0) {
            __nv_bfloat162 p2 = __floats2bfloat162_rn(h, h1);
            st_shared_b32(st + (uint32_t)j * 32u + (uint32_t)(lane >> 2) * 4u,
                          *reinterpret_cast<uint32_t*>(&p2));
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(mapC, st, f0, ti.row0 + c0);
          bulk_commit();
        }
        sbuf ^= 1;
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float x = __uint_as_float(v[j]);
          const float u = __shfl_xor_sync(0xffffffffu, x, 1);
          const int n = c0 + j;
          if (is_gate && n < ti.rows && f < a.F) {
            const float h = x / (1.0f + __expf(-x)) * u;
            a.out_bf16[(size_t)(ti.row0 + n) * a.F + f] = f_to_bf16(h);
          }
        }
      }
    }
  }
  // the tensor stores of this tile's H have completed before the count
  if (lane == 0) bulk_wait_all();
  __syncwarp();
  if (a.chunk_ready) {
    // this warp's H writes of the tile are visible before the count
    __threadfence();
    __syncwarp();
    if (lane == 0) atomicAdd(a.chunk_ready + ti.chunk, 1);
  }
}

}  // namespace dg
