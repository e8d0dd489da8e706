// Merge of the split-KV attention partials: for each canvas query row, the
// chunks' (O, m, l) (m in log2 units) combine by log-sum-exp into
// o = sum_c 2^{m_c - M} O_c / sum_c 2^{m_c - M} l_c, written as bf16 into the
// [T][Hq * dh] layout that the output projection reads.  One warp per row,
// lane c holding chunk c's (m, l) (at most 32 chunks).
#include "dg_kernels.h"

namespace dg {

namespace {

template <int DH>
__global__ void attn_merge_kernel(const AttnMergeArgs a, bf16* out) {
  griddep_wait();
  griddep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_total = a.B * a.Hq * a.Tc;
  const int R = blockIdx.x * (blockDim.x >> 5) + warp;
  if (R >= rows_total) return;
  // lane c holds chunk c's (m, l); n_chunks <= 32
  float mc = -INFINITY, lc = 0.f;
  if (lane < a.n_chunks) {
    const float2 ml = *reinterpret_cast<const float2*>(a.part_ml + ((size_t)lane * rows_total + R) * 2);
    mc = ml.x;
    lc = ml.y;
  }
  const float M = warp_max(mc);
  const float wl = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
  const float L = warp_sum(wl * lc);
  float acc[DH / 32];
#pragma unroll
  for (int j = 0; j < DH / 32; ++j) acc[j] = 0.f;
  for (int c = 0; c < a.n_chunks; ++c) {
    const float wgt = __shfl_sync(0xffffffffu, wl, c);
    const float* po = a.part_o + ((size_t)c * rows_total + R) * DH;
#pragma unroll
    for (int j = 0; j < DH / 32; ++j) acc[j] += wgt * po[lane + 32 * j];
  }
  const int i = R % a.Tc;
  const int bh = R / a.Tc;
  const int h = bh % a.Hq, b = bh / a.Hq;
  bf16* dst = out + ((size_t)b * a.Tc + i) * ((size_t)a.Hq * DH) + (size_t)h * DH;
  const float inv = 1.0f / L;
#pragma unroll
  for (int j = 0; j < DH / 32; ++j) dst[lane + 32 * j] = f_to_bf16(acc[j] * inv);
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
