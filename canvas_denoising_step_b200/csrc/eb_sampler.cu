// Entropy-bounded denoising on the device: the per-row entropy at a pass's
// temperature, and the per-canvas decisions of the pass (stop, bounded commit,
// inverse-CDF draw of the committed tokens).
//
// The vocab head GEMM (HEAD mode with inv_temp set) leaves, per token row and
// 256-wide vocab block, the block's max logit m_b, S_b = sum e^z and
// Q_b = sum z e^z with z = (l - m_b) / temp.  eb_merge folds the blocks into
// the row's max M, S = sum e^((l - M) / temp), its argmax and its entropy
// H = ln S - Q / S (nats, mask id excluded).  eb_commit then takes, per canvas:
//   stop   the mean entropy over all slots (summed in slot order, fp64) is below
//          the threshold and every argmax equals the previous pass's;
//   commit at a stop or at the last allowed pass, every masked slot takes its
//          argmax token; otherwise the masked slots in (entropy, slot) order are
//          committed while their running fp64 sum stays within the bound (at
//          least one), each with a token drawn by inverse CDF: the first vocab
//          index whose cumulative probability exceeds the slot's uniform u.
// The draw walks the block masses S_b e^((m_b - M) / temp) in vocab order to the
// block holding u * S, then recomputes that block's 256 logits (hn . E_v) and
// walks them.
#include "dg_kernels.h"

namespace dg {

namespace {

constexpr int kMergeWarps = 32;

__device__ __forceinline__ void merge_eb(float& m, float& s, float& q, int& a, float m2,
                                         float s2, float q2, int a2, float it) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) { m = m2; s = s2; q = q2; a = a2; return; }
  if (m2 > m) {
    const float d = (m - m2) * it, e = __expf(d);
    q = e * (q + d * s) + q2;
    s = e * s + s2;
    m = m2;
    a = a2;
  } else {
    const float d = (m2 - m) * it, e = __expf(d);
    q += e * (q2 + d * s2);
    s += e * s2;
    if (m2 == m && a2 < a) a = a2;
  }
}

// block-wide inclusive scan of one float per thread (256 threads)
__device__ __forceinline__ float block_incl_scan(float v, float* warp_tot) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  __syncthreads();
  if (lane == 31) warp_tot[w] = v;
  __syncthreads();
  float before = 0.f;
  for (int i = 0; i < w; ++i) before += warp_tot[i];
  return v + before;
}

}  // namespace

// ---------------------------------------------------------------- merge

__global__ void __launch_bounds__(kMergeWarps * 32) eb_merge_kernel(EbMergeArgs a) {
  __shared__ float s_m[kMergeWarps][32], s_s[kMergeWarps][32], s_q[kMergeWarps][32];
  __shared__ int s_a[kMergeWarps][32];
  griddep_wait();
  griddep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 32 + lane;
  const float it = *a.inv_temp;
  float m = -INFINITY, s = 0.f, q = 0.f;
  int arg = 0x7fffffff;
  if (t < a.T) {
    const int per = (a.n_vblocks + kMergeWarps - 1) / kMergeWarps;
    const int v0 = warp * per, v1 = min(a.n_vblocks, v0 + per);
    int vb = v0;
    for (; vb + 4 <= v1; vb += 4) {   // four blocks' loads in flight
      float mm[4], ss[4], qq[4];
      int aa[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const size_t o = (size_t)(vb + u) * a.T + t;
        mm[u] = a.hm[o];
        ss[u] = a.hs[o];
        qq[u] = a.hq[o];
        aa[u] = a.ha[o];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) merge_eb(m, s, q, arg, mm[u], ss[u], qq[u], aa[u], it);
    }
    for (; vb < v1; ++vb) {
      const size_t o = (size_t)vb * a.T + t;
      merge_eb(m, s, q, arg, a.hm[o], a.hs[o], a.hq[o], a.ha[o], it);
    }
  }
  s_m[warp][lane] = m;
  s_s[warp][lane] = s;
  s_q[warp][lane] = q;
  s_a[warp][lane] = arg;
  __syncthreads();
  if (warp == 0 && t < a.T) {
    float mt = -INFINITY, st = 0.f, qt = 0.f;
    int at = 0x7fffffff;
    for (int w = 0; w < kMergeWarps; ++w)
      merge_eb(mt, st, qt, at, s_m[w][lane], s_s[w][lane], s_q[w][lane], s_a[w][lane], it);
    a.H[t] = __logf(st) - qt / st;
    a.tok[t] = at;
    a.max_logit[t] = mt;
    a.sum[t] = st;
  }
}

cudaError_t launch_eb_merge(const EbMergeArgs& a, cudaStream_t s) {
  return launch_k(eb_merge_kernel, dim3((a.T + 31) / 32), dim3(kMergeWarps * 32), 0, s, a);
}

// ---------------------------------------------------------------- commit

__global__ void __launch_bounds__(256) eb_commit_kernel(EbCommitArgs a) {
  __shared__ float s_H[256];
  __shared__ int s_masked[256];
  __shared__ int s_by_rank[256];
  __shared__ int s_n_commit, s_stop, s_last;
  __shared__ float s_warp[8];
  __shared__ int s_pick;
  __shared__ float s_before;
  extern __shared__ __align__(16) uint8_t s_dyn[];   // hn row: d bf16
  griddep_wait();
  griddep_launch();
  const int b = blockIdx.x, i = threadIdx.x, Tc = a.Tc;
  const size_t o = (size_t)b * Tc;
  const int state = a.state ? a.state[b] : 0;      // bit 0: previous argmax kept, bit 1: done
  if (state & 2) {
    if (i < Tc && a.committed) a.committed[o + i] = 0;
    return;
  }
  int masked = 0, am = 0;
  float h = 0.f;
  bool same = true;
  if (i < Tc) {
    masked = a.canvas[o + i] == a.mask_id;
    h = a.H[o + i];
    am = a.argmax[o + i];
    const bool have_prev = a.prev_in && (a.state == nullptr || (state & 1));
    same = have_prev && a.prev_in[o + i] == am;
  }
  s_H[i] = h;
  s_masked[i] = masked;
  const int n_masked = __syncthreads_count(masked);
  const bool stable = __syncthreads_and(i < Tc ? same : true) && a.prev_in &&
                      (a.state == nullptr || (state & 1));
  if (i == 0) {
    double total = 0.0;
    for (int j = 0; j < Tc; ++j) total += (double)s_H[j];
    s_stop = (total / Tc < a.threshold) && stable;
    s_last = a.last_flag ? *a.last_flag : a.last;
  }
  __syncthreads();
  const bool all = s_stop || s_last;
  int rank = 0x7fffffff;
  if (!all && masked) {
    rank = 0;
    for (int j = 0; j < Tc; ++j)
      rank += s_masked[j] && (s_H[j] < h || (s_H[j] == h && j < i));
    s_by_rank[rank] = i;
  }
  __syncthreads();
  if (i == 0) {
    int n = 0;
    if (!all) {
      double total = 0.0;
      for (int r = 0; r < n_masked; ++r) {
        total += (double)s_H[s_by_rank[r]];
        if (r > 0 && total > a.bound) break;
        n = r + 1;
      }
    }
    s_n_commit = n;
  }
  __syncthreads();
  const int n_commit = s_n_commit;
  int com = 0;
  if (i < Tc && masked && all) {
    a.canvas[o + i] = am;
    com = 1;
  }
  // the committed slots' tokens, one slot at a time with the whole CTA
  bf16* hrow = reinterpret_cast<bf16*>(s_dyn);
  for (int r = 0; r < n_commit; ++r) {
    const int slot = s_by_rank[r];
    const size_t t = o + slot;
    int tok;
    if (a.drawn_in) {
      tok = a.drawn_in[t];
    } else {
      const float it = *a.inv_temp;
      const float M = a.max_logit[t];
      const float target = a.u[t] * a.sum[t];
      // 1) the vocab block: masses in vocab order, `per` consecutive blocks a thread
      const int per = (a.n_vblocks + 255) / 256;
      const int v0 = i * per, v1 = min(a.n_vblocks, v0 + per);
      float mine = 0.f;
      for (int vb = v0; vb < v1; ++vb) {
        const float mb = a.head_m[(size_t)vb * a.T + t];
        if (mb != -INFINITY) mine += a.head_s[(size_t)vb * a.T + t] * __expf((mb - M) * it);
      }
      const float incl = block_incl_scan(mine, s_warp);
      if (i == 0) s_pick = -1;
      __syncthreads();
      const float excl = incl - mine;
      if (v1 > v0 && excl <= target && target < incl) s_pick = i;   // at most one thread
      __syncthreads();
      int pick = s_pick;
      __syncthreads();   // every thread has read the pick before it is overwritten
      int vb_pick = -1;
      float before = 0.f;
      if (pick < 0) pick = min(255, (a.n_vblocks - 1) / per);   // rounding: the last range
      if (i == pick) {
        float acc = excl;
        for (int vb = v0; vb < v1; ++vb) {
          const float mb = a.head_m[(size_t)vb * a.T + t];
          const float mass = mb != -INFINITY ? a.head_s[(size_t)vb * a.T + t] * __expf((mb - M) * it) : 0.f;
          if (mass > 0.f) { vb_pick = vb; before = acc; }
          if (mass > 0.f && acc + mass > target) break;
          acc += mass;
        }
        s_pick = vb_pick;
        s_before = before;
      }
      __syncthreads();
      vb_pick = s_pick;
      before = s_before;
      tok = a.argmax[t];   // kept only if no vocab entry carries mass (cannot happen in exact arithmetic)
      if (vb_pick >= 0) {
        // 2) that block's logits, one vocab row a thread, then the walk inside it
        for (int c = i; c < a.d / 8; c += 256)
          reinterpret_cast<uint4*>(hrow)[c] = reinterpret_cast<const uint4*>(a.hn + t * a.d)[c];
        __syncthreads();
        // warp w computes the logits of vocab rows w*32 .. w*32+31 of the block, one
        // row at a time with the whole warp (coalesced reads of the embedding row,
        // a fixed-order warp sum); thread i keeps the logit of row i
        float l_mine = 0.f;
        const int warp = i >> 5, lane = i & 31;
        for (int rr = 0; rr < 32; ++rr) {
          const int vr = vb_pick * 256 + warp * 32 + rr;
          float part = 0.f;
          if (vr < a.vocab && vr != a.mask_id) {
            const uint4* er = reinterpret_cast<const uint4*>(a.embed + (size_t)vr * a.d);
            for (int c = lane; c < a.d / 8; c += 32) {
              const uint4 ev = er[c], hv = reinterpret_cast<const uint4*>(hrow)[c];
              const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w}, hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                part = fmaf(__uint_as_float(ew[k] << 16), __uint_as_float(hw[k] << 16), part);
                part = fmaf(__uint_as_float(ew[k] & 0xFFFF0000u), __uint_as_float(hw[k] & 0xFFFF0000u), part);
              }
            }
          }
          part = warp_sum(part);
          if (lane == rr) l_mine = part;
        }
        const int vid = vb_pick * 256 + i;
        float e = 0.f;
        if (vid < a.vocab && vid != a.mask_id) e = __expf((l_mine - M) * it);
        const float ci = block_incl_scan(e, s_warp);
        if (i == 0) s_pick = -1;
        __syncthreads();
        if (e > 0.f && before + ci > target && before + ci - e <= target) s_pick = i;   // one thread
        __syncthreads();
        if (s_pick < 0) {   // rounding: the last entry of the block with a non-zero mass
          __syncthreads();
          if (e > 0.f) atomicMax(&s_pick, i);
          __syncthreads();
        }
        if (s_pick >= 0) tok = vb_pick * 256 + s_pick;
      }
      __syncthreads();
    }
    if (i == 0) {
      a.canvas[t] = tok;
      if (a.drawn_out) a.drawn_out[t] = tok;
    }
    if (i == slot) com = 1;
    __syncthreads();
  }
  __syncthreads();
  if (i < Tc) {
    if (a.committed) a.committed[o + i] = (uint8_t)com;
    if (a.prev_out) a.prev_out[o + i] = am;
  }
  const int left = __syncthreads_count(i < Tc && a.canvas[o + i] == a.mask_id);
  if (i == 0) {
    if (a.stopped) a.stopped[b] = (uint8_t)s_stop;
    if (a.state_out) a.state_out[b] = 1 | ((s_stop || s_last || left == 0) ? 2 : 0);
  }
}

cudaError_t launch_eb_commit(const EbCommitArgs& a, cudaStream_t s) {
  if (a.Tc > 256 || a.d % 8) return cudaErrorInvalidValue;
  return launch_k(eb_commit_kernel, dim3(a.B), dim3(256), (size_t)a.d * 2, s, a);
}

__global__ void set_float_kernel(float* p, float v) { *p = v; }

cudaError_t launch_set_float(float* p, float v, cudaStream_t s) {
  set_float_kernel<<<1, 1, 0, s>>>(p, v);
  return cudaGetLastError();
}

}  // namespace dg
