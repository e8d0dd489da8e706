// Merge of the split-KV attention partials: for each canvas query row, the
// chunks' (O, m, l) (m in log2 units) combine by log-sum-exp into
// o = sum_c 2^{m_c - M} O_c / sum_c 2^{m_c - M} l_c, written as bf16 into the
// [T][Hq * dh] layout that the output projection reads.  One warp per row,
// lane c holding chunk c's (m, l) (at most 32 chunks).  Every rounding is
// explicit (no contraction), so the attention kernel's in-cluster merge, which
// takes the same steps in the same order, gives the same bits.
#include "dg_kernels.h"

namespace dg {

namespace {

template <int DH>
__global__ void attn_merge_kernel(const AttnMergeArgs a, bf16* out) {
  constexpr int NJ = DH / 64;   // float2 per lane per chunk: lane covers 2 * lane + 64 * j
  constexpr int kBatch = 4;     // chunks whose loads are in flight together
  griddep_wait();
  griddep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_total = a.B * a.Hq * a.Tc;
  const int R = blockIdx.x * (blockDim.x >> 5) + warp;
  if (R >= rows_total) return;
  const int nc = a.n_chunks;
  // lane c holds chunk c's (m, l); n_chunks <= 32
  float mc = -INFINITY, lc = 0.f;
  if (lane < nc) {
    const float2 ml = __ldcg(reinterpret_cast<const float2*>(a.part_ml + ((size_t)lane * rows_total + R) * 2));
    mc = ml.x;
    lc = ml.y;
  }
  float2 acc[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) acc[j] = make_float2(0.f, 0.f);
  float M = 0.f, wl = 0.f, L = 0.f;
  for (int c0 = 0; c0 < nc; c0 += kBatch) {
    // the partial O of up to kBatch chunks, loaded before they are needed
    float2 buf[kBatch][NJ];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
#pragma unroll
      for (int j = 0; j < NJ; ++j)
        buf[u][j] = (c0 + u < nc)
                        ? __ldcg(reinterpret_cast<const float2*>(
                              a.part_o + ((size_t)(c0 + u) * rows_total + R) * DH + 2 * lane + 64 * j))
                        : make_float2(0.f, 0.f);
    if (c0 == 0) {
      M = warp_max(mc);
      wl = (mc == -INFINITY) ? 0.f : exp2f(__fsub_rn(mc, M));
      L = warp_sum(__fmul_rn(wl, lc));
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const float wgt = __shfl_sync(0xffffffffu, wl, (c0 + u) & 31);
      if (c0 + u < nc)
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          acc[j].x = __fmaf_rn(wgt, buf[u][j].x, acc[j].x);
          acc[j].y = __fmaf_rn(wgt, buf[u][j].y, acc[j].y);
        }
    }
  }
  const int i = R % a.Tc;
  const int bh = R / a.Tc;
  const int h = bh % a.Hq, b = bh / a.Hq;
  bf16* dst = out + ((size_t)b * a.Tc + i) * ((size_t)a.Hq * DH) + (size_t)h * DH;
  const float inv = __frcp_rn(L);
#pragma unroll
  for (int j = 0; j < NJ; ++j)
    *reinterpret_cast<__nv_bfloat162*>(dst + 2 * lane + 64 * j) =
        __floats2bfloat162_rn(__fmul_rn(acc[j].x, inv), __fmul_rn(acc[j].y, inv));
}

}  // namespace

cudaError_t launch_attn_merge(const AttnMergeArgs& a, bf16* o, cudaStream_t s) {
  const int rows = a.B * a.Hq * a.Tc;
  const int grid = (rows + 7) / 8;
  switch (a.dh) {
    case 64: return launch_k(attn_merge_kernel<64>, dim3(grid), dim3(256), 0, s, a, o);
    case 128: return launch_k(attn_merge_kernel<128>, dim3(grid), dim3(256), 0, s, a, o);
    case 256: return launch_k(attn_merge_kernel<256>, dim3(grid), dim3(256), 0, s, a, o);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dg
