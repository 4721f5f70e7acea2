// decode.cuh -- single-step pi-attention decode for bf16 caches, head size 64 or 128.
//
// One new query per (b, h) reads its window (k_win + 1 contiguous cache rows ending at its own
// position) and its periodic skip rows, ~1 KB of cache per row pair and no reuse: the kernel is a
// pure HBM stream.  Layout of the work: a CTA of 2 warps per (b, h, split).  A row of d bf16 is
// read by d/8 lanes with one 16-byte load each, so a warp instruction covers 32*16 = 512
// contiguous bytes (2 rows at d = 128, 4 at d = 64) and every 32-byte sector is used whole.  Each
// group of d/8 lanes ("slot") keeps its own online-softmax state (running max m, sum l and 8
// accumulator columns) in the log2 domain; slots, warps and splits merge by the usual rescale
//   M = max(m_a, m_b),  l = l_a 2^(m_a - M) + l_b 2^(m_b - M),  acc likewise,
// which is the single softmax over the union evaluated in pieces.  With one split the CTA writes
// out/lse directly; with several, each split writes (m, l, acc) to a workspace and a second
// kernel merges them.
//
// The cache is either plain (position j in row j, len <= n_cache) or a ring of capacity
// C = n_cache (position j in slot j mod C, any len >= 1): a ring of C >= max(k, S pi) + 1 slots
// holds every key a decode step can still read, and a step appends one row (pi_attn_cache_append).
#pragma once
#include "common.cuh"

namespace pia {

struct DecodeArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* kc;
  const __nv_bfloat16* vc;
  const float* w_g;
  const float* b_g;
  const int* cache_len;
  __nv_bfloat16* out;
  float* lse;
  float* part;  // [B*H, nsplit, D + 2] when nsplit > 1: acc[D], m, l
  int H, n_cache, kwin, pi, S, nsplit;
  float scale_log2;
  int ring;     // 1: n_cache is the capacity of a ring cache (position j in slot j mod n_cache)
};

template <int D>
__device__ __forceinline__ void decode_merge(float& m, float& l, float* acc, float m2, float l2, const float* acc2) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;  // both empty
  const float c1 = exp2f(m - mn), c2 = exp2f(m2 - mn);
  l = l * c1 + l2 * c2;
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = acc[e] * c1 + acc2[e] * c2;
  m = mn;
}

template <int D>
// 14 CTAs an SM (at most 72 registers a thread): one wave holds 14 x 148 = 2072 CTAs, so a step
// of up to 2072 (b, h) runs in a single wave instead of one and a fraction.
__global__ void __launch_bounds__(64, 14) decode_bf16_kernel(DecodeArgs a) {
  constexpr int LPR = D / 8;      // lanes per cache row
  constexpr int RPI = 32 / LPR;   // rows per warp instruction
  constexpr int NW = 2;           // warps per CTA
  constexpr int UNR = 4;          // rows per slot per iteration (loads in flight)
  static_assert(D == 64 || D == 128, "decode kernel covers d = 64 and d = 128");

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % LPR, slot = lane / LPR;
  const long long bh = blockIdx.x;
  const int split = blockIdx.y;
  const int b = (int)(bh / a.H), h = (int)(bh % a.H);

  const int len = a.cache_len ? a.cache_len[b] : a.n_cache;
  if (len < 1 || (!a.ring && len > a.n_cache)) {
    if (split == 0) {
      if (threadIdx.x == 0) {
        raise_error(kErrCacheLen);
        if (a.lse) a.lse[bh] = __int_as_float(0x7fffffff);
      }
      for (int c = threadIdx.x; c < D; c += blockDim.x)
        a.out[bh * D + c] = __float2bfloat16_rn(__int_as_float(0x7fffffff));
    }
    if (a.nsplit > 1 && threadIdx.x == 0) {  // mark the split empty so the merge stays defined
      float* p = a.part + (bh * a.nsplit + split) * (D + 2);
      p[D] = -INFINITY;
      p[D + 1] = 0.f;
    }
    if (a.nsplit > 1)
      for (int c = threadIdx.x; c < D; c += blockDim.x) a.part[(bh * a.nsplit + split) * (D + 2) + c] = 0.f;
    return;
  }
  const long long i = len - 1;
  // window rows [j0, i]; skip rows i - m*pi for m = m0 .. m1 (those that exist)
  const long long j0 = i - a.kwin > 0 ? i - a.kwin : 0;
  const int nL = (int)(i - j0 + 1);
  const int m0 = first_skip_m(a.kwin, a.pi);
  long long m1 = i / a.pi;
  if (m1 > a.S) m1 = a.S;
  const int nP = m1 >= m0 ? (int)(m1 - m0 + 1) : 0;
  const int R = nL + nP;
  // ring: slots of the first window row and of the query row (one modulo each; window rows then
  // step forward and skip rows step back with at most one wrap, as k + 1 <= C and S pi < C)
  const long long C = a.n_cache;
  const long long j0s = a.ring ? j0 % C : j0, is = a.ring ? i % C : i;
  // this split's share of the R rows
  const int per = (R + a.nsplit - 1) / a.nsplit;
  const int t_begin = split * per;
  const int t_end = min(R, t_begin + per);

  // query slice and the gate
  const __nv_bfloat16* qrow = a.q + bh * D;
  float qf[8];
  bf16x8_to_f32(*reinterpret_cast<const uint4*>(qrow + sub * 8), qf);
  float z = 0.f;
  if (slot == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) z = fmaf(qf[e], a.w_g[(long long)h * D + sub * 8 + e], z);
  }
  z = warp_sum(z) + a.b_g[h];
  const float bias_l = log_sigmoid(z) * kLog2e;
  const float bias_p = log_sigmoid(-z) * kLog2e;

  const __nv_bfloat16* kb = a.kc + bh * (long long)a.n_cache * D + sub * 8;
  const __nv_bfloat16* vb = a.vc + bh * (long long)a.n_cache * D + sub * 8;

  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;

  // The trip count is the same for every lane of a warp (the loop variable is warp-uniform), so
  // the full-warp shuffles of the dot-product reduction always see all 32 lanes.
  constexpr int STEP = NW * RPI * UNR;
  for (int base = t_begin + warp * RPI * UNR; base < t_end; base += STEP) {
    const int t0 = base + slot * UNR;  // rows t0 .. t0+UNR-1 belong to this slot
    uint4 kr[UNR], vr[UNR];
    bool ok[UNR];
    float bias[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int t = t0 + u;
      ok[u] = t < t_end;
      long long j = t < nL ? j0s + t : is - (long long)(m0 + (t - nL)) * a.pi;  // cache row (slot)
      if (j >= C) j -= C;
      else if (j < 0) j += C;
      bias[u] = t < nL ? bias_l : bias_p;
      if (!ok[u]) j = is;  // a row that exists; its score is discarded below
      kr[u] = __ldg(reinterpret_cast<const uint4*>(kb + j * D));
      vr[u] = __ldg(reinterpret_cast<const uint4*>(vb + j * D));
    }
    float s[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      float kf[8];
      bf16x8_to_f32(kr[u], kf);
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(qf[e], kf[e], dot);
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      s[u] = ok[u] ? fmaf(dot, a.scale_log2, bias[u]) : -INFINITY;
    }
    float mn = m;
#pragma unroll
    for (int u = 0; u < UNR; ++u) mn = fmaxf(mn, s[u]);
    if (mn != -INFINITY) {  // per-slot state update; no warp-collective operation inside
      const float corr = exp2f(m - mn);
      l *= corr;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] *= corr;
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const float p = exp2f(s[u] - mn);
        l += p;
        float vf[8];
        bf16x8_to_f32(vr[u], vf);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(p, vf[e], acc[e]);
      }
      m = mn;
    }
  }

  // merge the slots of this warp (lanes with equal `sub`)
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
    float a2[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) a2[e] = __shfl_xor_sync(0xffffffffu, acc[e], o);
    decode_merge<D>(m, l, acc, m2, l2, a2);
  }
  // merge the two warps
  __shared__ float sm_acc[NW][D];
  __shared__ float sm_ml[NW][2];
  if (slot == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) sm_acc[warp][sub * 8 + e] = acc[e];
    if (sub == 0) {
      sm_ml[warp][0] = m;
      sm_ml[warp][1] = l;
    }
  }
  __syncthreads();
  if (warp == 0 && slot == 0) {
    float a2[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) a2[e] = sm_acc[1][sub * 8 + e];
    decode_merge<D>(m, l, acc, sm_ml[1][0], sm_ml[1][1], a2);
    if (a.nsplit == 1) {
      const float inv = 1.f / l;
      __align__(16) __nv_bfloat16 o8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) o8[e] = __float2bfloat16_rn(acc[e] * inv);
      *reinterpret_cast<uint4*>(a.out + bh * D + sub * 8) = *reinterpret_cast<const uint4*>(o8);
      if (sub == 0 && a.lse) a.lse[bh] = (m + log2f(l)) * kLn2;
    } else {
      float* p = a.part + (bh * a.nsplit + split) * (D + 2);
#pragma unroll
      for (int e = 0; e < 8; ++e) p[sub * 8 + e] = acc[e];
      if (sub == 0) {
        p[D] = m;
        p[D + 1] = l;
      }
    }
  }
}

// Merge the per-split partial states of each (b, h): one CTA of D threads per (b, h).
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const float* __restrict__ part, int nsplit,
                                                           const int* __restrict__ cache_len, int H, int n_cache,
                                                           __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                                                           int ring) {
  const long long bh = blockIdx.x;
  const int c = threadIdx.x;
  const int len = cache_len ? cache_len[bh / H] : n_cache;
  if (len < 1 || (!ring && len > n_cache)) return;  // already reported and written as NaN
  const float* p = part + bh * nsplit * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, p[s * (D + 2) + D]);
  float L = 0.f, acc = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float ms = p[s * (D + 2) + D];
    if (ms == -INFINITY) continue;
    const float w = exp2f(ms - M);
    L = fmaf(p[s * (D + 2) + D + 1], w, L);
    acc = fmaf(p[s * (D + 2) + c], w, acc);
  }
  out[bh * D + c] = __float2bfloat16_rn(acc / L);
  if (c == 0 && lse) lse[bh] = (M + log2f(L)) * kLn2;
}

// One decode step's new token into the cache: row cache_len[b] (mod C for a ring) of every
// (b, h) takes k_new / v_new; one CTA per (b, h), 16-byte chunks.  A cache_len below zero, or past
// C for a plain cache, sets the error word and writes nothing.
template <typename T>
__global__ void cache_append_kernel(T* __restrict__ kc, T* __restrict__ vc, const T* __restrict__ k_new,
                                    const T* __restrict__ v_new, const int* __restrict__ cache_len, int H, int C,
                                    int d, int ring) {
  const long long bh = blockIdx.x;
  const int b = (int)(bh / H);
  const int len = cache_len[b];
  if (len < 0 || (!ring && len >= C)) {
    if (threadIdx.x == 0) raise_error(kErrCacheLen);
    return;
  }
  const long long slot = ring ? len % C : len;
  const int vec = 16 / (int)sizeof(T);
  for (int c = threadIdx.x * vec; c < d; c += blockDim.x * vec) {
    *reinterpret_cast<uint4*>(kc + (bh * C + slot) * d + c) = *reinterpret_cast<const uint4*>(k_new + bh * d + c);
    *reinterpret_cast<uint4*>(vc + (bh * C + slot) * d + c) = *reinterpret_cast<const uint4*>(v_new + bh * d + c);
  }
}

// After every (b, h) of a step has been written: the lengths move on by one.
__global__ void cache_len_advance_kernel(int* __restrict__ cache_len, int B, int C, int ring) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B && cache_len[b] >= 0 && (ring || cache_len[b] < C)) cache_len[b] += 1;
}

}  // namespace pia
