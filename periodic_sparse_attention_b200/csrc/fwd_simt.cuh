// fwd_simt.cuh -- CUDA-core pi-attention: one warp per query row.
//
// The general path: every dtype (fp32, bf16) and head size up to 256, prefill and decode.  It is
// the fp32 path of the operator and the fallback for bf16 shapes the tensor-core kernel does not
// cover.  Per query row it walks the window keys, then the skip keys, with an online softmax in
// the log2 domain (scores pre-multiplied by tau*log2(e), priors by log2(e)), so the union is
// normalised by one running max and one running sum -- a single softmax over L(i) and P(i).
// `bidir` (prefill only) selects the bidirectional rule: the window reaches k tokens both ways
// and each m has a forward skip i + m*pi as well, up to the sequence end.
#pragma once
#include "common.cuh"

namespace pia {

template <typename T, bool DECODE>
__global__ void __launch_bounds__(256) simt_attn_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ w_g,
    const float* __restrict__ b_g, const int* __restrict__ cache_len, T* __restrict__ out, float* __restrict__ lse,
    int B, int H, int n_q, int n_kv, int d, int kwin, int pi, int S, float scale_log2, bool bidir) {
  const int lane = threadIdx.x & 31;
  const long long task = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long long ntask = DECODE ? (long long)B * H : (long long)B * H * n_q;
  if (task >= ntask) return;

  long long bh;
  long long i;
  const T* qrow;
  if (DECODE) {
    bh = task;
    const int b = (int)(bh / H);
    const int len = cache_len ? cache_len[b] : n_kv;
    if (len < 1 || len > n_kv) {
      if (lane == 0) {
        raise_error(kErrCacheLen);
        if (lse) lse[bh] = __int_as_float(0x7fffffff);
      }
      for (int c = lane; c < d; c += 32) out[bh * d + c] = from_f32<T>(__int_as_float(0x7fffffff));
      return;
    }
    i = len - 1;
    qrow = q + bh * d;
  } else {
    bh = task / n_q;
    i = task % n_q;
    qrow = q + task * d;
  }
  const int h = (int)(bh % H);
  const T* kb = k + bh * (long long)n_kv * d;
  const T* vb = v + bh * (long long)n_kv * d;

  float qr[8], acc[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int c = lane + 32 * u;
    qr[u] = c < d ? to_f32(qrow[c]) : 0.f;
    acc[u] = 0.f;
  }
  // gate on the unscaled query: z = q . w_g[h] + b_g[h]
  float z = 0.f;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int c = lane + 32 * u;
    if (c < d) z = fmaf(qr[u], w_g[(long long)h * d + c], z);
  }
  z = warp_sum(z) + b_g[h];
  const float bias_l = log_sigmoid(z) * kLog2e;   // log2(alpha)
  const float bias_p = log_sigmoid(-z) * kLog2e;  // log2(1 - alpha)

  float m = -INFINITY, l = 0.f;
  auto visit = [&](long long j, float bias) {
    const T* kr = kb + j * d;
    const T* vr = vb + j * d;
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = lane + 32 * u;
      if (c < d) s = fmaf(qr[u], to_f32(kr[c]), s);
    }
    s = fmaf(warp_sum(s), scale_log2, bias);
    const float mn = fmaxf(m, s);
    const float corr = exp2f(m - mn);
    const float p = exp2f(s - mn);
    l = fmaf(l, corr, p);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = lane + 32 * u;
      if (c < d) acc[u] = fmaf(acc[u], corr, p * to_f32(vr[c]));
    }
    m = mn;
  };
  const long long j0 = i - kwin > 0 ? i - kwin : 0;
  const long long j1 = bidir ? (i + kwin < n_kv - 1 ? i + kwin : n_kv - 1) : i;
  for (long long j = j0; j <= j1; ++j) visit(j, bias_l);
  for (long long mm = first_skip_m(kwin, pi); mm <= S; ++mm) {
    const long long jb = i - mm * pi, jf = i + mm * pi;
    if (jb >= 0) visit(jb, bias_p);
    if (bidir && jf < n_kv) visit(jf, bias_p);
    if (jb < 0 && (!bidir || jf >= n_kv)) break;
  }

  const float inv = 1.f / l;
  const long long orow = DECODE ? bh : task;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int c = lane + 32 * u;
    if (c < d) out[orow * d + c] = from_f32<T>(acc[u] * inv);
  }
  if (lse && lane == 0) lse[orow] = (m + log2f(l)) * kLn2;
}

// Index sets exactly as the kernels enumerate them (window ascending, then skips by m; for each m
// the backward key before the forward one).
__global__ void index_sets_kernel(int n, int kwin, int pi, int S, int width, bool bidir, int* __restrict__ counts,
                                  int* __restrict__ idx) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const long long j0 = i - kwin > 0 ? i - kwin : 0;
  const long long j1 = bidir ? (i + kwin < n - 1 ? i + kwin : n - 1) : i;
  int w = 0;
  int* row = idx + i * width;
  for (long long j = j0; j <= j1; ++j)
    if (w < width) row[w++] = (int)j;
  const int nl = (int)(j1 - j0 + 1);
  int np = 0;
  for (long long mm = first_skip_m(kwin, pi); mm <= S; ++mm) {
    const long long jb = i - mm * pi, jf = i + mm * pi;
    if (jb >= 0) {
      if (w < width) row[w++] = (int)jb;
      ++np;
    }
    if (bidir && jf < n) {
      if (w < width) row[w++] = (int)jf;
      ++np;
    }
    if (jb < 0 && (!bidir || jf >= n)) break;
  }
  while (w < width) row[w++] = -1;
  counts[2 * i] = nl;
  counts[2 * i + 1] = np;
}

}  // namespace pia
