// Weight initialisation on the device: the SplitMix64 counter generator with a
// four-term Irwin-Hall normal, written into the physical layouts of the weights.
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

}  // namespace dg
