// Element-wise, normalisation, routing, merge and commit kernels of the canvas step.
#include "dg_kernels.h"

namespace dg {

namespace {

constexpr unsigned long long kGamma = 0x9E3779B97F4A7C15ull;
constexpr unsigned long long kKeyMult = 0xD1B54A32D192ED03ull;

__host__ __device__ __forceinline__ unsigned long long mix64(unsigned long long z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Element `idx` of the stream with key `key`: the (idx+1)-th SplitMix64
// output, four 16-bit fields summed and centred (Irwin-Hall), times `scale`.
__device__ __forceinline__ bf16 gen_weight(unsigned long long key, unsigned long long idx,
                                           float scale) {
  const unsigned long long u = mix64(key + (idx + 1ull) * kGamma);
  const int s = (int)(u & 0xFFFFull) + (int)((u >> 16) & 0xFFFFull) +
                (int)((u >> 32) & 0xFFFFull) + (int)(u >> 48);
  const float x = __fmul_rn((float)(s - 131070), scale);
  return __float2bfloat16_rn(x);
}

constexpr int kMaxPerThread = 16;  // d <= 256 * 16

__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  const int nw = (blockDim.x + 31) >> 5;
  for (int i = 0; i < nw; ++i) t += red[i];
  return t;
}

}  // namespace

unsigned long long stream_key_host(unsigned long long seed, unsigned long long tid) {
  return mix64(seed + tid * kKeyMult);
}

// ---------------------------------------------------------------- weight init

__global__ void init_kernel(InitArgs a) {
  const long long base = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (base >= a.n_elems) return;
  bf16 out[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const long long p = base + e;
    unsigned long long key, idx;
    if (a.layout == INIT_PLAIN) {
      key = a.key0;
      idx = (unsigned long long)p;
    } else if (a.layout == INIT_QKV) {
      const long long row = p / a.cols, col = p % a.cols;
      if (row < a.rows_a) {
        key = a.key0; idx = (unsigned long long)(row * a.cols + col);
      } else if (row < a.rows_a + a.rows_b) {
        key = a.key1; idx = (unsigned long long)((row - a.rows_a) * a.cols + col);
      } else {
        key = a.key2; idx = (unsigned long long)((row - a.rows_a - a.rows_b) * a.cols + col);
      }
    } else if (a.layout == INIT_GATEUP) {
      const long long per_g = 2ll * a.F * a.d;
      const long long g = p / per_g, rem = p % per_g;
      const long long prow = rem / a.d, col = rem % a.d;
      const long long f = prow >> 1;
      const bool up = (prow & 1) != 0;
      if (g > 0) {  // routed expert g - 1
        key = up ? a.key1 : a.key0;
        idx = (unsigned long long)(((g - 1) * a.F + f) * a.d + col);
      } else {      // group 0: the shared expert
        key = up ? a.key3 : a.key2;
        idx = (unsigned long long)(f * a.d + col);
      }
    } else {  // INIT_DOWN
      const long long per_g = (long long)a.d * a.F;
      const long long g = p / per_g, rem = p % per_g;
      if (g > 0) { key = a.key0; idx = (unsigned long long)((g - 1) * per_g + rem); }
      else { key = a.key1; idx = (unsigned long long)rem; }
    }
    out[e] = gen_weight(key, idx, a.scale);
  }
  if (base + 3 < a.n_elems) {
    uint2 pk;
    pk.x = (uint32_t)__bfloat16_as_ushort(out[0]) | ((uint32_t)__bfloat16_as_ushort(out[1]) << 16);
    pk.y = (uint32_t)__bfloat16_as_ushort(out[2]) | ((uint32_t)__bfloat16_as_ushort(out[3]) << 16);
    *reinterpret_cast<uint2*>(a.dst + base) = pk;
  } else {
    for (int e = 0; e < 4 && base + e < a.n_elems; ++e) a.dst[base + e] = out[e];
  }
}

cudaError_t launch_init(const InitArgs& a, cudaStream_t s) {
  const long long threads = (a.n_elems + 3) / 4;
  const int bs = 256;
  const long long grid = (threads + bs - 1) / bs;
  init_kernel<<<(unsigned)grid, bs, 0, s>>>(a);
  return cudaGetLastError();
}

__global__ void fill_f32_kernel(float* p, long long n, float v) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}

cudaError_t launch_fill_f32(float* p, long long n, float v, cudaStream_t s) {
  fill_f32_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p, n, v);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- embed + input norm

__global__ void embed_norm_kernel(const int32_t* canvas, const bf16* embed, const bf16* x_in,
                                  int vocab, int d, const float* w, float eps, float* h, bf16* x,
                                  int* err) {
  __shared__ float red[32];
  const int t = blockIdx.x;
  const bf16* src;
  if (x_in) {
    src = x_in + (size_t)t * d;
  } else {
    int tok = canvas[t];
    if (tok < 0 || tok >= vocab) { raise_error(err, kErrFault); tok = 0; }
    src = embed + (size_t)tok * d;
  }
  float v[kMaxPerThread];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxPerThread; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    v[i] = (c < d) ? bf16_to_f(src[c]) : 0.f;
    ss += v[i] * v[i];
  }
  ss = block_sum(ss, red);
  const float r = rsqrtf(ss / (float)d + eps);
#pragma unroll
  for (int i = 0; i < kMaxPerThread; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    if (c < d) {
      h[(size_t)t * d + c] = v[i];
      x[(size_t)t * d + c] = f_to_bf16(v[i] * r * w[c]);
    }
  }
}

cudaError_t launch_embed_norm(const int32_t* canvas, const bf16* embed, const bf16* x_in,
                              int vocab, int T, int d, const float* w, float eps, float* h,
                              bf16* x, int* err, cudaStream_t s) {
  embed_norm_kernel<<<T, 256, 0, s>>>(canvas, embed, x_in, vocab, d, w, eps, h, x, err);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- RoPE

__global__ void rope_table_kernel(float* cos_t, float* sin_t, int Tc, int half, int P,
                                  double theta) {
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
  rope_table_kernel<<<(n + 255) / 256, 256, 0, s>>>(cos_t, sin_t, Tc, half, P, theta);
  return cudaGetLastError();
}

// One block per canvas row.  Thread u handles the pairs (head, j) numbered
// threadIdx.x + 256 * u; split-K partials are summed split by split so that
// each thread's loads of one split are independent of one another.
constexpr int kRopeMaxPerThread = 32;   // (Hq + 2 Hkv) * dh / 2 <= 8192

__global__ void __launch_bounds__(256) qkv_rope_kernel(const float* part, int splits, int T,
                                                       int Tc, int Hq, int Hkv, int dh, int n_rot,
                                                       const float* cos_t, const float* sin_t,
                                                       bf16* q, bf16* kc, bf16* vc) {
  const int t = blockIdx.x;
  const int b = t / Tc, i = t % Tc;
  const int nqkv = (Hq + 2 * Hkv) * dh;
  const int half = dh / 2;
  const int npairs = nqkv / 2;
  float x0[kRopeMaxPerThread], x1[kRopeMaxPerThread];
#pragma unroll
  for (int u = 0; u < kRopeMaxPerThread; ++u) x0[u] = x1[u] = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float* src = part + ((size_t)s * T + t) * nqkv;
#pragma unroll
    for (int u = 0; u < kRopeMaxPerThread; ++u) {
      const int p = threadIdx.x + 256 * u;
      if (p < npairs) {
        const int hh = p / half, j = p % half;
        x0[u] += src[hh * dh + j];
        x1[u] += src[hh * dh + j + half];
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kRopeMaxPerThread; ++u) {
    const int p = threadIdx.x + 256 * u;
    if (p >= npairs) continue;
    const int hh = p / half, j = p % half;
    bf16* dst;
    bool rotate = true;
    if (hh < Hq) dst = q + (((size_t)b * Hq + hh) * Tc + i) * dh;
    else if (hh < Hq + Hkv) dst = kc + (((size_t)b * Hkv + (hh - Hq)) * Tc + i) * dh;
    else { dst = vc + (((size_t)b * Hkv + (hh - Hq - Hkv)) * Tc + i) * dh; rotate = false; }
    float a0 = x0[u], a1 = x1[u];
    if (rotate && j < n_rot) {
      const float c = cos_t[i * half + j], sn = sin_t[i * half + j];
      const float y0 = a0 * c - a1 * sn;
      const float y1 = a0 * sn + a1 * c;
      a0 = y0;
      a1 = y1;
    }
    dst[j] = f_to_bf16(a0);
    dst[j + half] = f_to_bf16(a1);
  }
}

cudaError_t launch_qkv_rope(const float* part, int splits, int T, int Tc, int Hq, int Hkv, int dh,
                            int n_rot, const float* cos_t, const float* sin_t, bf16* q, bf16* kc,
                            bf16* vc, cudaStream_t s) {
  qkv_rope_kernel<<<T, 256, 0, s>>>(part, splits, T, Tc, Hq, Hkv, dh, n_rot, cos_t, sin_t, q, kc,
                                    vc);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- post-attention norms

__global__ void post_attn_kernel(const float* part, int splits, int T, int d, const float* w_post,
                                 const float* w_ff, float eps, float* h, bf16* x2) {
  __shared__ float red[32];
  const int t = blockIdx.x;
  float a[kMaxPerThread];
#pragma unroll
  for (int i = 0; i < kMaxPerThread; ++i) a[i] = 0.f;
  for (int s = 0; s < splits; ++s) {       // independent loads within one split
    const float* src = part + ((size_t)s * T + t) * d;
#pragma unroll
    for (int i = 0; i < kMaxPerThread; ++i) {
      const int c = threadIdx.x + i * blockDim.x;
      if (c < d) a[i] += src[c];
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxPerThread; ++i) ss += a[i] * a[i];
  ss = block_sum(ss, red);
  const float r1 = rsqrtf(ss / (float)d + eps);
  float ss2 = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxPerThread; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    if (c < d) {
      const float v = h[(size_t)t * d + c] + a[i] * r1 * w_post[c];
      a[i] = v;
      h[(size_t)t * d + c] = v;
      ss2 += v * v;
    }
  }
  ss2 = block_sum(ss2, red);
  const float r2 = rsqrtf(ss2 / (float)d + eps);
#pragma unroll
  for (int i = 0; i < kMaxPerThread; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    if (c < d) x2[(size_t)t * d + c] = f_to_bf16(a[i] * r2 * w_ff[c]);
  }
}

cudaError_t launch_post_attn(const float* part, int splits, int T, int d, const float* w_post,
                             const float* w_ff, float eps, float* h, bf16* x2, cudaStream_t s) {
  post_attn_kernel<<<T, 256, 0, s>>>(part, splits, T, d, w_post, w_ff, eps, h, x2);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- router

// One warp per row.  Selection by (logit desc, index asc); weights = softmax
// over the chosen logits; membership bits for the counting sort.
__global__ void router_topk_kernel(const float* part, int splits, const float* bias, int T, int E,
                                   int k, float* logits_out, int32_t* idx, float* w,
                                   uint32_t* bitmap) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= T) return;
  const int W = (T + 31) / 32;
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = 0.f;
  for (int s = 0; s < splits; ++s) {       // independent loads within one split
    const float* src = part + ((size_t)s * T + t) * E;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (e < E) v[i] += src[e];
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    float x = -INFINITY;
    if (e < E) {
      x = v[i];
      if (bias) x += bias[e];
      if (logits_out) logits_out[(size_t)t * E + e] = x;
      if (x != x) x = -INFINITY;
    }
    v[i] = x;
  }
  unsigned taken = 0;
  __shared__ float s_sel_v[8][32];
  __shared__ int s_sel_i[8][32];
  float* sel_v = s_sel_v[warp];
  int* sel_i = s_sel_i[warp];
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
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
    if (bi >= 0 && bi < E && (bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == 0) {
      sel_v[j] = bv;
      sel_i[j] = bi;
    }
  }
  __syncwarp();
  if (lane == 0) {
    const float mx = sel_v[0];
    float den = 0.f;
    for (int j = 0; j < k; ++j) den += __expf(sel_v[j] - mx);
    for (int j = 0; j < k; ++j) {
      int e = sel_i[j];
      if (e < 0 || e >= E) e = 0;
      idx[(size_t)t * k + j] = e;
      w[(size_t)t * k + j] = __expf(sel_v[j] - mx) / den;
      atomicOr(bitmap + (size_t)e * W + (t >> 5), 1u << (t & 31));
    }
  }
}

cudaError_t launch_router_topk(const float* part, int splits, const float* bias, int T, int E,
                               int k, float* logits_out, int32_t* idx, float* w,
                               uint32_t* bitmap, cudaStream_t s) {
  const int rows_per_block = 8;
  router_topk_kernel<<<(T + rows_per_block - 1) / rows_per_block, 32 * rows_per_block, 0, s>>>(
      part, splits, bias, T, E, k, logits_out, idx, w, bitmap);
  return cudaGetLastError();
}

cudaError_t launch_router_topk_only(const float* logits, int T, int E, int k, int32_t* idx,
                                    float* w, uint32_t* bitmap, cudaStream_t s) {
  return launch_router_topk(logits, 1, nullptr, T, E, k, nullptr, idx, w, bitmap, s);
}

// Single CTA counting sort, stable in row order.  prefix[e*W + w] = number of
// rows < 32w assigned to e.  Routed positions p are relative (0 .. T*k-1);
// in the permuted activation buffer the routed row p sits at T + p, after
// the T rows of the shared-expert group 0.
__global__ void router_sort_kernel(const int32_t* idx, uint32_t* bitmap, int T, int E, int k,
                                   int n_shared, int n_tile, int32_t* offsets_r,
                                   int32_t* offsets_g, int32_t* chunk_prefix, int32_t* perm,
                                   int32_t* inv, int* err, int* active_out) {
  extern __shared__ int sm[];
  const int W = (T + 31) / 32;
  int* prefix = sm;              // [E*W]
  int* count = sm + E * W;       // [E]
  int* off = count + E;          // [E+1]
  for (int i = threadIdx.x; i < E * W; i += blockDim.x) prefix[i] = __popc(bitmap[i]);
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
  if (threadIdx.x == 0) {
    int run = 0;
    int crun = n_shared ? (T + n_tile - 1) / n_tile : 0;
    if (offsets_g) { offsets_g[0] = 0; }
    if (chunk_prefix) { chunk_prefix[0] = 0; chunk_prefix[1] = crun; }
    for (int e = 0; e < E; ++e) {
      off[e] = run;
      if (offsets_r) offsets_r[e] = run;
      if (offsets_g) offsets_g[e + 1] = T + run;
      run += count[e];
      crun += (count[e] + n_tile - 1) / n_tile;
      if (chunk_prefix) chunk_prefix[e + 2] = crun;
    }
    off[E] = run;
    if (offsets_r) offsets_r[E] = run;
    if (active_out) {
      int active = 0;
      for (int e = 0; e < E; ++e) active += count[e] > 0;
      atomicAdd(active_out, active);
    }
    if (offsets_g) offsets_g[E + 1] = T + run;
    if (run != T * k) raise_error(err, kErrFault);
  }
  __syncthreads();
  for (int a = threadIdx.x; a < T * k; a += blockDim.x) {
    const int t = a / k;
    const int e = idx[a];
    if (e < 0 || e >= E) { raise_error(err, kErrFault); continue; }
    const uint32_t word = bitmap[(size_t)e * W + (t >> 5)];
    const int pos = off[e] + prefix[e * W + (t >> 5)] + __popc(word & ((1u << (t & 31)) - 1u));
    perm[pos] = a;
    inv[a] = pos;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E * W; i += blockDim.x) bitmap[i] = 0u;
}

cudaError_t launch_router_sort(const int32_t* idx, uint32_t* bitmap, int T, int E, int k,
                               int n_shared, int n_tile, int32_t* offsets_r, int32_t* offsets_g,
                               int32_t* chunk_prefix, int32_t* perm, int32_t* inv, int* err,
                               int* active_out, cudaStream_t s) {
  const int W = (T + 31) / 32;
  const size_t smem = (size_t)(E * W + E + E + 1) * sizeof(int);
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(router_sort_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  router_sort_kernel<<<1, 1024, smem, s>>>(idx, bitmap, T, E, k, n_shared, n_tile, offsets_r,
                                           offsets_g, chunk_prefix, perm, inv, err, active_out);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- MoE gather / combine

__global__ void moe_gather_kernel(bf16* xperm, const int32_t* perm, int T, int k, int d) {
  const int p = blockIdx.x;
  const int t = perm[p] / k;
  const uint4* src = reinterpret_cast<const uint4*>(xperm + (size_t)t * d);
  uint4* dst = reinterpret_cast<uint4*>(xperm + ((size_t)T + p) * d);
  for (int i = threadIdx.x; i < d / 8; i += blockDim.x) dst[i] = src[i];
}

cudaError_t launch_moe_gather(bf16* xperm, const int32_t* perm, int T, int k, int d,
                              cudaStream_t s) {
  moe_gather_kernel<<<T * k, 128, 0, s>>>(xperm, perm, T, k, d);
  return cudaGetLastError();
}

__global__ void moe_combine_kernel(const float* Y, const float* w, const int32_t* inv, int T,
                                   int k, int n_shared, int d, float* h, const float* w_next,
                                   float eps, bf16* x) {
  __shared__ float red[32];
  __shared__ int srow[33];
  __shared__ float sw[33];
  const int t = blockIdx.x;
  if (threadIdx.x < k) {
    srow[threadIdx.x] = T + inv[(size_t)t * k + threadIdx.x];
    sw[threadIdx.x] = w[(size_t)t * k + threadIdx.x];
  }
  __syncthreads();
  float v[kMaxPerThread];
#pragma unroll
  for (int i = 0; i < kMaxPerThread; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    v[i] = (c < d) ? h[(size_t)t * d + c] : 0.f;
  }
  float y[kMaxPerThread];
#pragma unroll
  for (int i = 0; i < kMaxPerThread; ++i) y[i] = 0.f;
  for (int j = 0; j < k; ++j) {            // fixed order j = 0 .. k-1
    const float* src = Y + (size_t)srow[j] * d;
    const float wj = sw[j];
#pragma unroll
    for (int i = 0; i < kMaxPerThread; ++i) {
      const int c = threadIdx.x + i * blockDim.x;
      if (c < d) y[i] += wj * src[c];
    }
  }
  if (n_shared) {
    const float* src = Y + (size_t)t * d;
#pragma unroll
    for (int i = 0; i < kMaxPerThread; ++i) {
      const int c = threadIdx.x + i * blockDim.x;
      if (c < d) y[i] += src[c];
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxPerThread; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    v[i] += y[i];
    if (c < d) h[(size_t)t * d + c] = v[i];
    ss += v[i] * v[i];
  }
  if (w_next) {
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / (float)d + eps);
#pragma unroll
    for (int i = 0; i < kMaxPerThread; ++i) {
      const int c = threadIdx.x + i * blockDim.x;
      if (c < d) x[(size_t)t * d + c] = f_to_bf16(v[i] * r * w_next[c]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < kMaxPerThread; ++i) {
      const int c = threadIdx.x + i * blockDim.x;
      if (c < d) x[(size_t)t * d + c] = f_to_bf16(v[i]);
    }
  }
}

cudaError_t launch_moe_combine(const float* Y, const float* w, const int32_t* inv, int T, int k,
                               int n_shared, int d, float* h, const float* w_next, float eps,
                               bf16* x, cudaStream_t s) {
  moe_combine_kernel<<<T, 256, 0, s>>>(Y, w, inv, T, k, n_shared, d, h, w_next, eps, x);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- vocab head merge

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

__global__ void head_merge_kernel(const float* hm, const float* hs, const int* ha, int n_vblocks,
                                  int T, float* conf, int32_t* tok) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= T) return;
  float m = -INFINITY, s = 0.f;
  int a = 0x7fffffff;
  const int per = (n_vblocks + 31) / 32;
  const int v0 = lane * per, v1 = min(n_vblocks, v0 + per);
  for (int vb = v0; vb < v1; ++vb) {
    const size_t o = (size_t)vb * T + t;
    merge_stats(m, s, a, hm[o], hs[o], ha[o]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    const int a2 = __shfl_xor_sync(0xffffffffu, a, o);
    merge_stats(m, s, a, m2, s2, a2);
  }
  if (lane == 0) {
    conf[t] = 1.0f / s;
    tok[t] = a;
  }
}

cudaError_t launch_head_merge(const float* hm, const float* hs, const int* ha, int n_vblocks,
                              int T, float* conf, int32_t* tok, cudaStream_t s) {
  head_merge_kernel<<<(T + 7) / 8, 256, 0, s>>>(hm, hs, ha, n_vblocks, T, conf, tok);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- commit

__global__ void commit_kernel(const float* conf, const int32_t* tok, int32_t* canvas,
                              uint8_t* committed, int Tc, int steps_left, const int* steps_dev,
                              int mask_id) {
  __shared__ float sc[256];
  __shared__ int sm[256];
  const int b = blockIdx.x, i = threadIdx.x;
  const size_t o = (size_t)b * Tc;
  int masked = 0;
  if (i < Tc) {
    masked = canvas[o + i] == mask_id;
    float c = conf[o + i];
    if (c != c) c = -INFINITY;
    sc[i] = c;
    sm[i] = masked;
  }
  const int r = __syncthreads_count(masked);
  const int sl = steps_left >= 1 ? steps_left : max(1, *steps_dev);
  const int k = (r + sl - 1) / sl;
  if (i < Tc) {
    int com = 0;
    if (masked) {
      const float ci = sc[i];
      int rank = 0;
      for (int j = 0; j < Tc; ++j)
        rank += sm[j] && (sc[j] > ci || (sc[j] == ci && j < i));
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
  commit_kernel<<<B, 256, 0, s>>>(conf, tok, canvas, committed, Tc, steps_left, steps_left_dev,
                                  mask_id);
  return cudaGetLastError();
}

}  // namespace dg
