// bwd_simt.cuh -- the backward of pi-attention on CUDA cores: gradients of a loss through out.
//
// The forward is recomputed, not stored: every kernel takes q, k, v, w_g, b_g and dO only.  With
// p_ij the softmax weight of key j for row i (one softmax over L(i) and P(i)), dO_i = dLoss/dout_i:
//   D_i  = dO_i . out_i,   dp_ij = dO_i . v_j,   ds_ij = p_ij (dp_ij - D_i)
//   dq_i = tau sum_j ds_ij k_j + dz_i w_g[h]             (the gate reads the unscaled query)
//   dk_j = tau sum_i ds_ij q_i,   dv_j = sum_i p_ij dO_i
//   dz_i = (1 - alpha_i) sum_{j in L(i)} ds_ij - alpha_i sum_{j in P(i)} ds_ij
//   dw_g[h] = sum_{b,i} dz_i q_i,   db_g[h] = sum_{b,i} dz_i
// Three kernels, no atomics (the result does not depend on scheduling):
//   bwd_row_kernel   one warp per query row: the row's softmax and output (online, fp32), D_i,
//                    then dq_i and dz_i; saves lse_i, D_i, the two log2-priors and dz_i per row
//   bwd_key_kernel   one warp per key row j: walks the rows that read key j (the index rule read
//                    backwards) and accumulates dk_j and dv_j
//   bwd_gate_*       dw_g and db_g, summed over rows in chunks and then over chunks, in a fixed order
// Gradients are fp32 whatever the storage type of the inputs.
#pragma once
#include "common.cuh"

namespace pia {

// Per-row values the key kernel and the gate kernel read back (fp32, [B*H*n] each).
struct BwdRowStats {
  float* lse2;  // log2 of the row's softmax denominator (log2 units, as the logits)
  float* D;     // dO_i . out_i
  float* bl2;   // log2(alpha_i): the window prior
  float* bp2;   // log2(1 - alpha_i): the skip prior
  float* dz;    // dLoss / dz_i
};

// Visit the keys of row i in the oracle's order: window ascending, then skips by increasing m
// (the backward key before the forward one).  f(j, is_window).
template <typename F>
__device__ __forceinline__ void for_each_key(long long i, long long n, int kwin, int pi, int S, bool bidir, F&& f) {
  const long long j0 = i - kwin > 0 ? i - kwin : 0;
  const long long j1 = bidir ? (i + kwin < n - 1 ? i + kwin : n - 1) : i;
  for (long long j = j0; j <= j1; ++j) f(j, true);
  for (long long m = first_skip_m(kwin, pi); m <= S; ++m) {
    const long long jb = i - m * pi, jf = i + m * pi;
    if (jb >= 0) f(jb, false);
    if (bidir && jf < n) f(jf, false);
    if (jb < 0 && (!bidir || jf >= n)) break;
  }
}

// Visit the rows that read key j: row i reads j as a window key when j is in L(i), as a skip key
// when j is in P(i).  f(i, is_window).
template <typename F>
__device__ __forceinline__ void for_each_reader(long long j, long long n, int kwin, int pi, int S, bool bidir, F&& f) {
  const long long i0 = bidir ? (j - kwin > 0 ? j - kwin : 0) : j;
  const long long i1 = j + kwin < n - 1 ? j + kwin : n - 1;
  for (long long i = i0; i <= i1; ++i) f(i, true);
  for (long long m = first_skip_m(kwin, pi); m <= S; ++m) {
    const long long ia = j + m * pi, ib = j - m * pi;  // rows after j read it backward; before it, forward
    if (ia < n) f(ia, false);
    if (bidir && ib >= 0) f(ib, false);
    if (ia >= n && (!bidir || ib < 0)) break;
  }
}

template <typename T>
__global__ void __launch_bounds__(256) bwd_row_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                      const T* __restrict__ v, const float* __restrict__ w_g,
                                                      const float* __restrict__ b_g, const T* __restrict__ dout,
                                                      float* __restrict__ dq, BwdRowStats st, int B, int H, int n,
                                                      int d, int kwin, int pi, int S, float scale_log2, bool bidir) {
  const int lane = threadIdx.x & 31;
  const long long task = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (task >= (long long)B * H * n) return;
  const long long bh = task / n, i = task % n;
  const int h = (int)(bh % H);
  const T* kb = k + bh * (long long)n * d;
  const T* vb = v + bh * (long long)n * d;
  float qr[8], gr[8], acc[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int c = lane + 32 * u;
    qr[u] = c < d ? to_f32(q[task * d + c]) : 0.f;
    gr[u] = c < d ? to_f32(dout[task * d + c]) : 0.f;
    acc[u] = 0.f;
  }
  float z = 0.f;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int c = lane + 32 * u;
    if (c < d) z = fmaf(qr[u], w_g[(long long)h * d + c], z);
  }
  z = warp_sum(z) + b_g[h];
  const float alpha = 1.f / (1.f + expf(-z));
  const float bl2 = log_sigmoid(z) * kLog2e, bp2 = log_sigmoid(-z) * kLog2e;

  auto logit = [&](long long j, bool win) {  // log2 units
    const T* kr = kb + j * d;
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = lane + 32 * u;
      if (c < d) s = fmaf(qr[u], to_f32(kr[c]), s);
    }
    return fmaf(warp_sum(s), scale_log2, win ? bl2 : bp2);
  };
  // the row's forward: one online softmax over the union, out_i in acc
  float m = -INFINITY, l = 0.f;
  for_each_key(i, n, kwin, pi, S, bidir, [&](long long j, bool win) {
    const float s = logit(j, win);
    const float mn = fmaxf(m, s);
    const float corr = exp2f(m - mn), p = exp2f(s - mn);
    l = fmaf(l, corr, p);
    const T* vr = vb + j * d;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = lane + 32 * u;
      if (c < d) acc[u] = fmaf(acc[u], corr, p * to_f32(vr[c]));
    }
    m = mn;
  });
  const float lse2 = m + log2f(l), inv = 1.f / l;
  float Dp = 0.f;
#pragma unroll
  for (int u = 0; u < 8; ++u) Dp = fmaf(gr[u], acc[u] * inv, Dp);
  const float D = warp_sum(Dp);
  // the row's backward
  float dqa[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) dqa[u] = 0.f;
  float dz = 0.f;
  for_each_key(i, n, kwin, pi, S, bidir, [&](long long j, bool win) {
    const float p = exp2f(logit(j, win) - lse2);
    const T* vr = vb + j * d;
    const T* kr = kb + j * d;
    float dp = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = lane + 32 * u;
      if (c < d) dp = fmaf(gr[u], to_f32(vr[c]), dp);
    }
    const float ds = p * (warp_sum(dp) - D);
    dz += win ? (1.f - alpha) * ds : -alpha * ds;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = lane + 32 * u;
      if (c < d) dqa[u] = fmaf(ds, to_f32(kr[c]), dqa[u]);
    }
  });
  const float tau = scale_log2 / kLog2e;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int c = lane + 32 * u;
    if (c < d) dq[task * d + c] = fmaf(tau, dqa[u], dz * w_g[(long long)h * d + c]);
  }
  if (lane == 0) {
    st.lse2[task] = lse2;
    st.D[task] = D;
    st.bl2[task] = bl2;
    st.bp2[task] = bp2;
    st.dz[task] = dz;
  }
}

template <typename T>
__global__ void __launch_bounds__(256) bwd_key_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                      const T* __restrict__ v, const T* __restrict__ dout,
                                                      BwdRowStats st, float* __restrict__ dk, float* __restrict__ dv,
                                                      int B, int H, int n, int d, int kwin, int pi, int S,
                                                      float scale_log2, bool bidir) {
  const int lane = threadIdx.x & 31;
  const long long task = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (task >= (long long)B * H * n) return;
  const long long bh = task / n, j = task % n;
  const long long rbase = bh * (long long)n;  // first row of this (b, h)
  float kr[8], vr[8], dka[8], dva[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int c = lane + 32 * u;
    kr[u] = c < d ? to_f32(k[task * d + c]) : 0.f;
    vr[u] = c < d ? to_f32(v[task * d + c]) : 0.f;
    dka[u] = dva[u] = 0.f;
  }
  for_each_reader(j, n, kwin, pi, S, bidir, [&](long long i, bool win) {
    const long long row = rbase + i;
    const T* qr = q + row * d;
    const T* gr = dout + row * d;
    float s = 0.f, dp = 0.f;
    float qv[8], gv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = lane + 32 * u;
      qv[u] = c < d ? to_f32(qr[c]) : 0.f;
      gv[u] = c < d ? to_f32(gr[c]) : 0.f;
      s = fmaf(qv[u], kr[u], s);
      dp = fmaf(gv[u], vr[u], dp);
    }
    s = fmaf(warp_sum(s), scale_log2, win ? st.bl2[row] : st.bp2[row]);
    const float p = exp2f(s - st.lse2[row]);
    const float ds = p * (warp_sum(dp) - st.D[row]);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      dva[u] = fmaf(p, gv[u], dva[u]);
      dka[u] = fmaf(ds, qv[u], dka[u]);
    }
  });
  const float tau = scale_log2 / kLog2e;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int c = lane + 32 * u;
    if (c < d) {
      dk[task * d + c] = tau * dka[u];
      dv[task * d + c] = dva[u];
    }
  }
}

// dw_g[h][c] = sum over (b, i) of dz * q[c], db_g[h] = sum of dz, in two stages with a fixed order:
// bwd_gate_partial_kernel sums chunks of kGateRows rows of one head (one block per (chunk, head),
// one thread per column), bwd_gate_final_kernel adds the chunks in increasing order.
constexpr int kGateRows = 32;

template <typename T>
__global__ void __launch_bounds__(256) bwd_gate_partial_kernel(const T* __restrict__ q, const float* __restrict__ dz,
                                                               float* __restrict__ part_w, float* __restrict__ part_b,
                                                               int B, int H, int n, int d) {
  const int chunk = blockIdx.x, h = blockIdx.y, nchunks = gridDim.x;
  const int c = threadIdx.x;
  const long long rows = (long long)B * n;  // rows of head h, in (b, i) order
  const long long t0 = (long long)chunk * kGateRows;
  const long long t1 = t0 + kGateRows < rows ? t0 + kGateRows : rows;
  float aw = 0.f, ab = 0.f;
  for (long long t = t0; t < t1; ++t) {
    const long long row = ((t / n) * H + h) * (long long)n + t % n;
    const float g = dz[row];
    if (c < d) aw = fmaf(g, to_f32(q[row * d + c]), aw);
    ab += g;
  }
  if (c < d) part_w[((long long)h * nchunks + chunk) * d + c] = aw;
  if (c == 0) part_b[(long long)h * nchunks + chunk] = ab;
}

__global__ void __launch_bounds__(256) bwd_gate_final_kernel(const float* __restrict__ part_w,
                                                             const float* __restrict__ part_b,
                                                             float* __restrict__ dw_g, float* __restrict__ db_g,
                                                             int nchunks, int d) {
  const int h = blockIdx.x, c = threadIdx.x;
  float aw = 0.f, ab = 0.f;
  for (int k = 0; k < nchunks; ++k) {
    if (c < d) aw += part_w[((long long)h * nchunks + k) * d + c];
    if (c == 0) ab += part_b[(long long)h * nchunks + k];
  }
  if (c < d) dw_g[(long long)h * d + c] = aw;
  if (c == 0) db_g[h] = ab;
}

}  // namespace pia
