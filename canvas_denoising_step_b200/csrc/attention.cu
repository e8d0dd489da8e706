// Canvas attention: one softmax over {the visible prompt keys} U {all canvas
// keys} for every canvas query row, grouped-query (Hq / Hkv query heads per
// key/value head), computed split-KV: each CTA takes 64 query rows of one
// (canvas, kv head) and one chunk of the key list, and writes the partial
// (O = sum_j 2^{s_j - m} v_j, m, l = sum_j 2^{s_j - m}) with s in log2 units;
// a merge kernel combines the chunks by log-sum-exp.
//
// This version runs QK^T and PV on the warp-level bf16 MMA (m16n8k16) with
// ldmatrix from 128-byte-XOR-swizzled shared memory, cp.async loads of the
// 64-key K/V blocks (single-buffered so that two CTAs share an SM and hide
// each other's loads), and the online softmax in registers.
#include "dg_kernels.h"

namespace dg {

namespace {

constexpr int kQRows = 64;   // query rows per CTA (4 warps x 16)
constexpr int kKeys = 64;    // keys per block

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// element offset of (row, col) in a [rows][DH] tile with 16-byte chunks XOR-swizzled by row % 8
template <int DH>
__device__ __forceinline__ int swz(int row, int col) {
  return row * DH + ((((col >> 3) ^ (row & 7))) << 3) + (col & 7);
}

template <int DH>
__global__ void __launch_bounds__(128, 2) attn_partial_kernel(const AttnArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  bf16* Qs = reinterpret_cast<bf16*>(smem_raw);
  bf16* Ks = Qs + kQRows * DH;         // [kKeys][DH]
  bf16* Vs = Ks + kKeys * DH;          // [kKeys][DH]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  griddep_wait();
  griddep_launch();
  const int qt = blockIdx.x, chunk = blockIdx.y;
  const int b = blockIdx.z / a.Hkv, g = blockIdx.z % a.Hkv;
  const int group = a.Hq / a.Hkv;
  const int q_rows = group * a.Tc;
  const int NK = a.n_vis + a.Tc;
  const int k_begin = chunk * a.chunk_keys;
  const int k_end = min(NK, k_begin + a.chunk_keys);
  const int rows_total = a.B * a.Hq * a.Tc;

  const bf16* qbase = a.q + ((size_t)b * a.Hq + (size_t)g * group) * a.Tc * DH;
  const bf16* kp = a.kp + ((size_t)b * a.Hkv + g) * a.P * DH;
  const bf16* vp = a.vp + ((size_t)b * a.Hkv + g) * a.P * DH;
  const bf16* kc = a.kc + ((size_t)b * a.Hkv + g) * a.Tc * DH;
  const bf16* vc = a.vc + ((size_t)b * a.Hkv + g) * a.Tc * DH;
  constexpr int CPR = DH / 8;  // 16-byte chunks per row

  // Q tile
  for (int c = tid; c < kQRows * CPR; c += 128) {
    const int r = c / CPR, q = c % CPR;
    const int qr = qt * kQRows + r;
    const bool valid = qr < q_rows;
    const bf16* src = qbase + (size_t)(valid ? qr : 0) * DH + q * 8;
    cp_async16(smem_u32(Qs + swz<DH>(r, q * 8)), src, valid);
  }
  auto load_kv = [&](int blk) {
    const int kb0 = k_begin + blk * kKeys;
    bf16* kd = Ks;
    bf16* vd = Vs;
    for (int c = tid; c < kKeys * CPR; c += 128) {
      const int j = c / CPR, q = c % CPR;
      const int kk = kb0 + j;
      const bool valid = kk < k_end;
      const bf16 *ks, *vs;
      if (!valid) { ks = kc; vs = vc; }
      else if (kk < a.n_vis) {
        const size_t row = (size_t)(a.P - a.n_vis + kk) * DH;
        ks = kp + row; vs = vp + row;
      } else {
        const size_t row = (size_t)(kk - a.n_vis) * DH;
        ks = kc + row; vs = vc + row;
      }
      cp_async16(smem_u32(kd + swz<DH>(j, q * 8)), ks + q * 8, valid);
      cp_async16(smem_u32(vd + swz<DH>(j, q * 8)), vs + q * 8, valid);
    }
  };

  const int n_blocks = (k_end > k_begin) ? (k_end - k_begin + kKeys - 1) / kKeys : 0;
  if (n_blocks > 0) load_kv(0);
  cp_async_commit();

  float o[DH / 8][4];
#pragma unroll
  for (int i = 0; i < DH / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int gq = lane >> 2, tq = lane & 3;

  for (int blk = 0; blk < n_blocks; ++blk) {
    if (blk > 0) {
      load_kv(blk);
      cp_async_commit();
    }
    cp_async_wait<0>();
    __syncthreads();
    const bf16* Kb = Ks;
    const bf16* Vb = Vs;

    // S = Q K^T for this warp's 16 rows x 64 keys
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < DH / 16; ++ks) {
      uint32_t af[4];
      {
        const int row = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = ks * 16 + (lane >> 4) * 8;
        ldsm_x4(smem_u32(Qs + swz<DH>(row, col)), af[0], af[1], af[2], af[3]);
      }
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int key = np * 16 + (lane & 7) + (lane >> 4) * 8;
        const int col = ks * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4(smem_u32(Kb + swz<DH>(key, col)), b0, b1, b2, b3);
        mma_bf16_16816(s[2 * np], af, b0, b1);
        mma_bf16_16816(s[2 * np + 1], af, b2, b3);
      }
    }
    // scale (log2 units), mask, online softmax
    const int kb0 = k_begin + blk * kKeys;
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kb0 + nt * 8 + 2 * tq + (e & 1);
        const float v = (key < k_end) ? s[nt][e] * a.scale_log2 : -INFINITY;
        s[nt][e] = v;
      }
      mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0;
    const float mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
    const float al0 = exp2f(m0 - mu0), al1 = exp2f(m1 - mu1);
    m0 = mn0;
    m1 = mn1;
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = exp2f(s[nt][0] - mu0);
      s[nt][1] = exp2f(s[nt][1] - mu0);
      s[nt][2] = exp2f(s[nt][2] - mu1);
      s[nt][3] = exp2f(s[nt][3] - mu1);
      rs0 += s[nt][0] + s[nt][1];
      rs1 += s[nt][2] + s[nt][3];
    }
    l0 = l0 * al0 + rs0;
    l1 = l1 * al1 + rs1;
#pragma unroll
    for (int i = 0; i < DH / 8; ++i) {
      o[i][0] *= al0; o[i][1] *= al0;
      o[i][2] *= al1; o[i][3] *= al1;
    }
    // O += P V
#pragma unroll
    for (int kv = 0; kv < kKeys / 16; ++kv) {
      uint32_t pf[4];
      pf[0] = pack_bf16(s[2 * kv][0], s[2 * kv][1]);
      pf[1] = pack_bf16(s[2 * kv][2], s[2 * kv][3]);
      pf[2] = pack_bf16(s[2 * kv + 1][0], s[2 * kv + 1][1]);
      pf[3] = pack_bf16(s[2 * kv + 1][2], s[2 * kv + 1][3]);
#pragma unroll
      for (int p = 0; p < DH / 16; ++p) {
        uint32_t b0, b1, b2, b3;
        const int key = kv * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = p * 16 + (lane >> 4) * 8;
        ldsm_x4_t(smem_u32(Vb + swz<DH>(key, col)), b0, b1, b2, b3);
        mma_bf16_16816(o[2 * p], pf, b0, b1);
        mma_bf16_16816(o[2 * p + 1], pf, b2, b3);
      }
    }
    __syncthreads();
  }

  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int qr = qt * kQRows + warp * 16 + gq + half * 8;
    if (qr >= q_rows) continue;
    const int h = g * group + qr / a.Tc, i = qr % a.Tc;
    const size_t R = ((size_t)b * a.Hq + h) * a.Tc + i;
    float* po = a.part_o + ((size_t)chunk * rows_total + R) * DH;
#pragma unroll
    for (int nt = 0; nt < DH / 8; ++nt) {
      float2 v = make_float2(o[nt][half * 2], o[nt][half * 2 + 1]);
      *reinterpret_cast<float2*>(po + nt * 8 + 2 * tq) = v;
    }
    if (tq == 0) {
      float* pml = a.part_ml + ((size_t)chunk * rows_total + R) * 2;
      pml[0] = half ? m1 : m0;
      pml[1] = half ? l1 : l0;
    }
  }
}

template <int DH>
__global__ void attn_merge_kernel(const AttnArgs a, bf16* out) {
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

template <int DH>
cudaError_t launch_attention_t(const AttnArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)(kQRows + 2 * kKeys) * DH * sizeof(bf16);
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_partial_kernel<DH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int group = a.Hq / a.Hkv;
  dim3 grid((group * a.Tc + kQRows - 1) / kQRows, a.n_chunks, a.B * a.Hkv);
  return launch_k(attn_partial_kernel<DH>, grid, dim3(128), smem, s, a);
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s) {
  switch (a.dh) {
    case 64: return launch_attention_t<64>(a, s);
    case 128: return launch_attention_t<128>(a, s);
    case 256: return launch_attention_t<256>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attn_merge(const AttnArgs& a, bf16* o, cudaStream_t s) {
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
