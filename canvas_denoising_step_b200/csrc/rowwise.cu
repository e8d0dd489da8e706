// Row-wise kernels of the canvas step: embedding + input norm, q/k RoPE,
// post-attention norm + residual + pre-FFN norm, MoE gather and combine,
// vocab-head merge and commit.
//
// Each row kernel runs one CTA of 256 threads per canvas row.  Thread i owns
// the 8-element chunks i and i + 256 of the row (d <= 4096), loaded as 16-byte
// vectors; the loads of several source rows (split-K partials, expert rows)
// are issued together before any of them is used, so a CTA keeps tens of KB in
// flight instead of one dependent round trip per source row.
#include <cstdlib>
#include <map>
#include <mutex>
#include <utility>

#include "dg_kernels.h"

namespace dg {

namespace {

constexpr int kRowThreads = 256;
constexpr int kChunks = 2;  // 8-element chunks per thread: d <= 256 * 2 * 8

__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < kRowThreads / 32; ++i) t += red[i];
  return t;
}

__device__ __forceinline__ void ld8f(const float* p, float* v) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// plain (coherent) loads for buffers written earlier in the same kernel chain
__device__ __forceinline__ void ld8f_rw(const float* p, float* v) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void st8f(float* p, const float* v) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

__device__ __forceinline__ void ld8b(const bf16* p, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ void st8b(bf16* p, const float* v) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&b);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace

cudaError_t ensure_smem_limit(const void* func, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> done;   // (kernel, device) -> bytes set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find({func, dev});
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  done[{func, dev}] = bytes;
  return cudaSuccess;
}

bool pdl_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("DG_NO_PDL");
    v = (e && e[0] && e[0] != '0') ? 0 : 1;
  }
  return v == 1;
}

// ---------------------------------------------------------------- embed + input norm

__global__ void __launch_bounds__(kRowThreads) embed_norm_kernel(
    const int32_t* canvas, const bf16* embed, const bf16* x_in, int vocab, int d, const float* w,
    float eps, float* h, bf16* x, int* err) {
  __shared__ float red[32];
  griddep_wait();
  griddep_launch();
  const int t = blockIdx.x;
  const bf16* src;
  if (x_in) {
    src = x_in + (size_t)t * d;
  } else {
    int tok = canvas[t];
    if (tok < 0 || tok >= vocab) { raise_error(err, kErrFault); tok = 0; }
    src = embed + (size_t)tok * d;
  }
  const int n8 = d / 8;
  float v[kChunks][8];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    const int c = threadIdx.x + kRowThreads * i;
    if (c < n8) ld8b(src + 8 * c, v[i]);
    else
#pragma unroll
      for (int e = 0; e < 8; ++e) v[i][e] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss += v[i][e] * v[i][e];
  }
  ss = block_sum(ss, red);
  const float r = rsqrtf(ss / (float)d + eps);
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    const int c = threadIdx.x + kRowThreads * i;
    if (c >= n8) continue;
    float wv[8], o[8];
    ld8f(w + 8 * c, wv);
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = v[i][e] * r * wv[e];
    st8f(h + (size_t)t * d + 8 * c, v[i]);
    st8b(x + (size_t)t * d + 8 * c, o);
  }
}

cudaError_t launch_embed_norm(const int32_t* canvas, const bf16* embed, const bf16* x_in,
                              int vocab, int T, int d, const float* w, float eps, float* h,
                              bf16* x, int* err, cudaStream_t s) {
  return launch_k(embed_norm_kernel, dim3(T), dim3(kRowThreads), 0, s, canvas, embed, x_in,
                  vocab, d, w, eps, h, x, err);
}

// ---------------------------------------------------------------- RoPE table

__global__ void rope_table_kernel(float* cos_t, float* sin_t, int Tc, int half, int P,
                                  double theta) {
  griddep_wait();
  griddep_launch();
  const int id = blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= Tc * half) return;
  const int i = id / half, j = id % half;
  const double inv_freq = pow(theta, -2.0 * (double)j / (double)(2 * half));
  const double ang = (double)(P + i) * inv_freq;
  double sn, cs;
  sincos(ang, &sn, &cs);
  cos_t[id] = (float)cs;
  sin_t[id] = (float)sn;
}

cudaError_t launch_rope_table(float* cos_t, float* sin_t, int Tc, int half, int P, double theta,
                              cudaStream_t s) {
  const int n = Tc * half;
  return launch_k(rope_table_kernel, dim3((n + 255) / 256), dim3(256), 0, s, cos_t, sin_t, Tc,
                  half, P, theta);
}

// ---------------------------------------------------------------- q/k/v split-K sum + RoPE

// A CTA takes one canvas row and up to kRopeThreads * kRopeItems work items of
// it (a second grid dimension covers wider rows).  Work item p = (head hh,
// 4-pair group j4): pairs (j, j + dh/2) for j = 4*j4 .. 4*j4+3, loaded as two
// float4 per split, two splits' loads in flight at once.  Four items per
// thread keep the registers low enough for two CTAs per SM.
constexpr int kRopeItems = 4;
constexpr int kRopeThreads = 256;

__global__ void __launch_bounds__(kRopeThreads, 2) qkv_rope_kernel(
    const float* part, int splits, int T, int Tc, int Hq, int Hkv, int dh, int n_rot,
    const float* cos_t, const float* sin_t, bf16* q, bf16* kc, bf16* vc) {
  griddep_wait();
  griddep_launch();
  const int t = blockIdx.x;
  const int b = t / Tc, i = t % Tc;
  const int nqkv = (Hq + 2 * Hkv) * dh;
  const int half = dh / 2, q4 = half / 4;
  const int n_items = (Hq + 2 * Hkv) * q4;
  const int p0 = blockIdx.y * kRopeThreads * kRopeItems + threadIdx.x;
  float4 x0[kRopeItems], x1[kRopeItems];
#pragma unroll
  for (int u = 0; u < kRopeItems; ++u) x0[u] = x1[u] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < splits; s0 += 2) {
    float4 a[2][kRopeItems], c[2][kRopeItems];
#pragma unroll
    for (int ss = 0; ss < 2; ++ss) {
      const float* src = part + ((size_t)(s0 + ss) * T + t) * nqkv;
#pragma unroll
      for (int u = 0; u < kRopeItems; ++u) {
        const int p = p0 + kRopeThreads * u;
        if (s0 + ss < splits && p < n_items) {
          const int hh = p / q4, j = (p % q4) * 4;
          a[ss][u] = __ldcg(reinterpret_cast<const float4*>(src + hh * dh + j));
          c[ss][u] = __ldcg(reinterpret_cast<const float4*>(src + hh * dh + j + half));
        } else {
          a[ss][u] = c[ss][u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
#pragma unroll
    for (int ss = 0; ss < 2; ++ss)
#pragma unroll
      for (int u = 0; u < kRopeItems; ++u) {
        x0[u].x += a[ss][u].x; x0[u].y += a[ss][u].y; x0[u].z += a[ss][u].z; x0[u].w += a[ss][u].w;
        x1[u].x += c[ss][u].x; x1[u].y += c[ss][u].y; x1[u].z += c[ss][u].z; x1[u].w += c[ss][u].w;
      }
  }
#pragma unroll
  for (int u = 0; u < kRopeItems; ++u) {
    const int p = p0 + kRopeThreads * u;
    if (p >= n_items) continue;
    const int hh = p / q4, j = (p % q4) * 4;
    bf16* dst;
    bool rotate = true;
    if (hh < Hq) dst = q + (((size_t)b * Hq + hh) * Tc + i) * dh;
    else if (hh < Hq + Hkv) dst = kc + (((size_t)b * Hkv + (hh - Hq)) * Tc + i) * dh;
    else { dst = vc + (((size_t)b * Hkv + (hh - Hq - Hkv)) * Tc + i) * dh; rotate = false; }
    float lo[4] = {x0[u].x, x0[u].y, x0[u].z, x0[u].w};
    float hi[4] = {x1[u].x, x1[u].y, x1[u].z, x1[u].w};
    if (rotate) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (j + e < n_rot) {
          const float cs = cos_t[i * half + j + e], sn = sin_t[i * half + j + e];
          const float y0 = lo[e] * cs - hi[e] * sn;
          const float y1 = lo[e] * sn + hi[e] * cs;
          lo[e] = y0;
          hi[e] = y1;
        }
      }
    }
    __nv_bfloat162 l01 = __floats2bfloat162_rn(lo[0], lo[1]), l23 = __floats2bfloat162_rn(lo[2], lo[3]);
    __nv_bfloat162 h01 = __floats2bfloat162_rn(hi[0], hi[1]), h23 = __floats2bfloat162_rn(hi[2], hi[3]);
    *reinterpret_cast<uint2*>(dst + j) =
        make_uint2(*reinterpret_cast<uint32_t*>(&l01), *reinterpret_cast<uint32_t*>(&l23));
    *reinterpret_cast<uint2*>(dst + j + half) =
        make_uint2(*reinterpret_cast<uint32_t*>(&h01), *reinterpret_cast<uint32_t*>(&h23));
  }
}

cudaError_t launch_qkv_rope(const float* part, int splits, int T, int Tc, int Hq, int Hkv, int dh,
                            int n_rot, const float* cos_t, const float* sin_t, bf16* q, bf16* kc,
                            bf16* vc, cudaStream_t s) {
  const int n_items = (Hq + 2 * Hkv) * (dh / 8);
  const int per_cta = kRopeThreads * kRopeItems;
  return launch_k(qkv_rope_kernel, dim3(T, (n_items + per_cta - 1) / per_cta), dim3(kRopeThreads),
                  0, s, part, splits, T, Tc, Hq, Hkv, dh, n_rot, cos_t, sin_t, q, kc, vc);
}

// ---------------------------------------------------------------- post-attention norms

__global__ void __launch_bounds__(kRowThreads) post_attn_kernel(
    const float* part, int splits, int T, int d, const float* w_post, const float* w_ff, float eps,
    float* h, bf16* x2) {
  __shared__ float red[32];
  griddep_wait();
  griddep_launch();
  const int t = blockIdx.x, n8 = d / 8;
  // the residual row goes out first, beside the partials' loads
  float hv[kChunks][8];
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    const int c = threadIdx.x + kRowThreads * i;
    if (c < n8) ld8f_rw(h + (size_t)t * d + 8 * c, hv[i]);
  }
  float a[kChunks][8];
#pragma unroll
  for (int i = 0; i < kChunks; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) a[i][e] = 0.f;
  for (int s0 = 0; s0 < splits; s0 += 4) {  // four splits' loads in flight at once
    float buf[4][kChunks][8];
#pragma unroll
    for (int ss = 0; ss < 4; ++ss)
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        const int c = threadIdx.x + kRowThreads * i;
        if (s0 + ss < splits && c < n8) ld8f(part + ((size_t)(s0 + ss) * T + t) * d + 8 * c, buf[ss][i]);
      }
#pragma unroll
    for (int ss = 0; ss < 4; ++ss)
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        const int c = threadIdx.x + kRowThreads * i;
        if (s0 + ss < splits && c < n8)
#pragma unroll
          for (int e = 0; e < 8; ++e) a[i][e] += buf[ss][i][e];
      }
  }
  float ss1 = 0.f;
#pragma unroll
  for (int i = 0; i < kChunks; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) ss1 += a[i][e] * a[i][e];
  ss1 = block_sum(ss1, red);
  const float r1 = rsqrtf(ss1 / (float)d + eps);
  float ss2 = 0.f;
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    const int c = threadIdx.x + kRowThreads * i;
    if (c >= n8) continue;
    float wv[8];
    ld8f(w_post + 8 * c, wv);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      a[i][e] = hv[i][e] + a[i][e] * r1 * wv[e];
      ss2 += a[i][e] * a[i][e];
    }
    st8f(h + (size_t)t * d + 8 * c, a[i]);
  }
  ss2 = block_sum(ss2, red);
  const float r2 = rsqrtf(ss2 / (float)d + eps);
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    const int c = threadIdx.x + kRowThreads * i;
    if (c >= n8) continue;
    float wv[8], o[8];
    ld8f(w_ff + 8 * c, wv);
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = a[i][e] * r2 * wv[e];
    st8b(x2 + (size_t)t * d + 8 * c, o);
  }
}

cudaError_t launch_post_attn(const float* part, int splits, int T, int d, const float* w_post,
                             const float* w_ff, float eps, float* h, bf16* x2, cudaStream_t s) {
  return launch_k(post_attn_kernel, dim3(T), dim3(kRowThreads), 0, s, part, splits, T, d, w_post,
                  w_ff, eps, h, x2);
}

// ---------------------------------------------------------------- MoE gather / combine

__global__ void moe_gather_kernel(bf16* xperm, const int32_t* perm, int T, int k, int d) {
  griddep_wait();
  griddep_launch();
  const int p = blockIdx.x;
  const int t = perm[p] / k;
  const uint4* src = reinterpret_cast<const uint4*>(xperm + (size_t)t * d);
  uint4* dst = reinterpret_cast<uint4*>(xperm + ((size_t)T + p) * d);
  // all of this thread's 16-byte pieces are loaded before any is stored
  constexpr int kPieces = 4;   // d / 8 <= 4 * 128 (d <= 4096)
  uint4 r[kPieces];
#pragma unroll
  for (int u = 0; u < kPieces; ++u) {
    const int i = threadIdx.x + (int)blockDim.x * u;
    if (i < d / 8) r[u] = src[i];
  }
#pragma unroll
  for (int u = 0; u < kPieces; ++u) {
    const int i = threadIdx.x + (int)blockDim.x * u;
    if (i < d / 8) dst[i] = r[u];
  }
}

cudaError_t launch_moe_gather(bf16* xperm, const int32_t* perm, int T, int k, int d,
                              cudaStream_t s) {
  return launch_k(moe_gather_kernel, dim3(T * k), dim3(128), 0, s, xperm, perm, T, k, d);
}

// y_t = sum_{j < k} w_tj Y[T + inv(t,j)] (+ Y[t] for the shared expert), added in
// the fixed order j = 0 .. k-1 then shared; h += y; then the next norm.
__global__ void __launch_bounds__(kRowThreads) moe_combine_kernel(
    const float* Y, const float* w, const int32_t* inv, int T, int k, int n_shared, int d, float* h,
    const float* w_next, float eps, bf16* x) {
  __shared__ float red[32];
  __shared__ int srow[33];
  __shared__ float sw[33];
  griddep_wait();
  griddep_launch();
  const int t = blockIdx.x, n8 = d / 8;
  // the residual row goes out with the routing loads
  float hv[kChunks][8];
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    const int c = threadIdx.x + kRowThreads * i;
    if (c < n8) ld8f_rw(h + (size_t)t * d + 8 * c, hv[i]);
  }
  if (threadIdx.x < k) {
    srow[threadIdx.x] = T + inv[(size_t)t * k + threadIdx.x];
    sw[threadIdx.x] = w[(size_t)t * k + threadIdx.x];
  }
  if (threadIdx.x == 0 && n_shared) {
    srow[k] = t;
    sw[k] = 1.0f;
  }
  __syncthreads();
  const int nrows = k + (n_shared ? 1 : 0);
  float y[kChunks][8];
#pragma unroll
  for (int i = 0; i < kChunks; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) y[i][e] = 0.f;
  for (int j0 = 0; j0 < nrows; j0 += 4) {     // four source rows' loads in flight at once
    float buf[4][kChunks][8];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        const int c = threadIdx.x + kRowThreads * i;
        if (j0 + jj < nrows && c < n8) ld8f_rw(Y + (size_t)srow[j0 + jj] * d + 8 * c, buf[jj][i]);
      }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      if (j0 + jj >= nrows) break;
      const float wj = sw[j0 + jj];
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        const int c = threadIdx.x + kRowThreads * i;
        if (c < n8)
#pragma unroll
          for (int e = 0; e < 8; ++e) y[i][e] += wj * buf[jj][i][e];
      }
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    const int c = threadIdx.x + kRowThreads * i;
    if (c >= n8) continue;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      y[i][e] += hv[i][e];
      ss += y[i][e] * y[i][e];
    }
    st8f(h + (size_t)t * d + 8 * c, y[i]);
  }
  if (w_next) {
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / (float)d + eps);
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
      const int c = threadIdx.x + kRowThreads * i;
      if (c >= n8) continue;
      float wv[8], o[8];
      ld8f(w_next + 8 * c, wv);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = y[i][e] * r * wv[e];
      st8b(x + (size_t)t * d + 8 * c, o);
    }
  } else {
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
      const int c = threadIdx.x + kRowThreads * i;
      if (c < n8) st8b(x + (size_t)t * d + 8 * c, y[i]);
    }
  }
}

cudaError_t launch_moe_combine(const float* Y, const float* w, const int32_t* inv, int T, int k,
                               int n_shared, int d, float* h, const float* w_next, float eps,
                               bf16* x, cudaStream_t s) {
  return launch_k(moe_combine_kernel, dim3(T), dim3(kRowThreads), 0, s, Y, w, inv, T, k, n_shared,
                  d, h, w_next, eps, x);
}

// ---------------------------------------------------------------- vocab head merge

namespace {
__device__ __forceinline__ void merge_stats(float& m, float& s, int& a, float m2, float s2,
                                            int a2) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) { m = m2; s = s2; a = a2; return; }
  if (m2 > m) {
    s = s * __expf(m - m2) + s2;
    m = m2;
    a = a2;
  } else {
    s = s + s2 * __expf(m2 - m);
    if (m2 == m && a2 < a) a = a2;
  }
}
}  // namespace

// A CTA takes 32 token rows (lane = row) and its 32 warps split the vocab
// blocks into contiguous slices, so that each load instruction reads 32
// consecutive rows of one block; warp 0 then merges the 32 slices of each row
// in slice order (the argmax tie rule, lowest index, does not depend on the
// order; the sum is taken in a fixed order).
constexpr int kMergeWarps = 32;

__global__ void __launch_bounds__(kMergeWarps * 32) head_merge_kernel(
    const float* hm, const float* hs, const int* ha, int n_vblocks, int T, float* conf,
    int32_t* tok, float* max_logit) {
  __shared__ float s_m[kMergeWarps][32], s_s[kMergeWarps][32];
  __shared__ int s_a[kMergeWarps][32];
  griddep_wait();
  griddep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 32 + lane;
  float m = -INFINITY, sum = 0.f;
  int arg = 0x7fffffff;
  if (t < T) {
    const int per = (n_vblocks + kMergeWarps - 1) / kMergeWarps;
    const int v0 = warp * per, v1 = min(n_vblocks, v0 + per);
    int vb = v0;
    for (; vb + 4 <= v1; vb += 4) {   // four blocks' loads in flight
      float mm[4], ss[4];
      int aa[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const size_t o = (size_t)(vb + u) * T + t;
        mm[u] = hm[o];
        ss[u] = hs[o];
        aa[u] = ha[o];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) merge_stats(m, sum, arg, mm[u], ss[u], aa[u]);
    }
    for (; vb < v1; ++vb) {
      const size_t o = (size_t)vb * T + t;
      merge_stats(m, sum, arg, hm[o], hs[o], ha[o]);
    }
  }
  s_m[warp][lane] = m;
  s_s[warp][lane] = sum;
  s_a[warp][lane] = arg;
  __syncthreads();
  if (warp == 0 && t < T) {
    float mt = -INFINITY, st = 0.f;
    int at = 0x7fffffff;
    for (int w = 0; w < kMergeWarps; ++w) merge_stats(mt, st, at, s_m[w][lane], s_s[w][lane], s_a[w][lane]);
    conf[t] = 1.0f / st;
    tok[t] = at;
    max_logit[t] = mt;
  }
}

cudaError_t launch_head_merge(const float* hm, const float* hs, const int* ha, int n_vblocks,
                              int T, float* conf, int32_t* tok, float* max_logit,
                              cudaStream_t s) {
  return launch_k(head_merge_kernel, dim3((T + 31) / 32), dim3(kMergeWarps * 32), 0, s, hm, hs,
                  ha, n_vblocks, T, conf, tok, max_logit);
}

// ---------------------------------------------------------------- commit

__global__ void commit_kernel(const float* conf, const int32_t* tok, int32_t* canvas,
                              uint8_t* committed, int Tc, int steps_left, const int* steps_dev,
                              int mask_id) {
  __shared__ __align__(16) float sc[256];
  __shared__ __align__(16) int sm[256];
  griddep_wait();
  griddep_launch();
  const int b = blockIdx.x, i = threadIdx.x;
  const size_t o = (size_t)b * Tc;
  const int sl = steps_left >= 1 ? steps_left : max(1, *steps_dev);
  int masked = 0;
  float c = -INFINITY;
  if (i < Tc) {
    masked = canvas[o + i] == mask_id;
    c = conf[o + i];
    if (c != c) c = -INFINITY;
  }
  sc[i] = c;          // slots past Tc: not masked, never counted
  sm[i] = masked;
  const int r = __syncthreads_count(masked);
  const int k = (r + sl - 1) / sl;
  if (i < Tc) {
    int com = 0;
    if (masked) {
      const float ci = c;
      int rank = 0;
      // four slots per shared-memory load
      for (int j = 0; j < Tc; j += 4) {
        const float4 c4 = *reinterpret_cast<const float4*>(sc + j);
        const int4 m4 = *reinterpret_cast<const int4*>(sm + j);
        rank += m4.x && (c4.x > ci || (c4.x == ci && j < i));
        rank += m4.y && (c4.y > ci || (c4.y == ci && j + 1 < i));
        rank += m4.z && (c4.z > ci || (c4.z == ci && j + 2 < i));
        rank += m4.w && (c4.w > ci || (c4.w == ci && j + 3 < i));
      }
      if (rank < k) {
        canvas[o + i] = tok[o + i];
        com = 1;
      }
    }
    if (committed) committed[o + i] = (uint8_t)com;
  }
}

cudaError_t launch_commit(const float* conf, const int32_t* tok, int32_t* canvas,
                          uint8_t* committed, int B, int Tc, int steps_left,
                          const int* steps_left_dev, int mask_id, cudaStream_t s) {
  return launch_k(commit_kernel, dim3(B), dim3(256), 0, s, conf, tok, canvas, committed, Tc,
                  steps_left, steps_left_dev, mask_id);
}

}  // namespace dg

namespace dg {

// ---------------------------------------------------------------- KV append

// Copy the new tokens' keys and values kc / vc [B][Hkv][n][dh] into the cache
// [B][Hkv][C][dh] at positions P0 .. P0 + n - 1: one warp per (b, head, token)
// row, 16 bytes per lane per step.
__global__ void kv_append_kernel(const bf16* __restrict__ kc, const bf16* __restrict__ vc,
                                 bf16* __restrict__ ck, bf16* __restrict__ cv, int rows, int n,
                                 int dh, int C, int P0) {
  griddep_wait();
  griddep_launch();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const int bg = warp / n, i = warp % n;
  const size_t src = (size_t)warp * dh;
  const size_t dst = ((size_t)bg * C + P0 + i) * dh;
  for (int e = lane * 8; e < dh; e += 32 * 8) {
    *reinterpret_cast<uint4*>(ck + dst + e) = *reinterpret_cast<const uint4*>(kc + src + e);
    *reinterpret_cast<uint4*>(cv + dst + e) = *reinterpret_cast<const uint4*>(vc + src + e);
  }
}

cudaError_t launch_kv_append(const bf16* kc, const bf16* vc, bf16* ck, bf16* cv, int B, int Hkv,
                             int n, int dh, int C, int P0, cudaStream_t s) {
  if (dh % 8 != 0 || P0 + n > C) return cudaErrorInvalidValue;
  const int rows = B * Hkv * n;
  return launch_k(kv_append_kernel, dim3((rows + 7) / 8), dim3(256), 0, s, kc, vc, ck, cv, rows, n,
                  dh, C, P0);
}

__global__ void set_int_kernel(int* p, int v) { *p = v; }

cudaError_t launch_set_int(int* p, int v, cudaStream_t s) {
  set_int_kernel<<<1, 1, 0, s>>>(p, v);
  return cudaGetLastError();
}

}  // namespace dg
