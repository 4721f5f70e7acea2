// bwd_simt.cuh -- the backward of pi-attention on CUDA cores: gradients of a loss through out.
//
// The forward is recomputed, not stored: every kernel takes q, k, v, w_g, b_g and dO only.  With
// p_ij the softmax weight of key j for row i (one softmax over L(i) and P(i)), dO_i = dLoss/dout_i:
//   D_i  = dO_i . out_i,   dp_ij = dO_i . v_j,   ds_ij = p_ij (dp_ij - D_i)
//   dq_i = tau sum_j ds_ij k_j + dz_i w_g[h]             (the gate reads the unscaled query)
//   dk_j = tau sum_i ds_ij q_i,   dv_j = sum_i p_ij dO_i
//   dz_i = (1 - alpha_i) sum_{j in L(i)} ds_ij - alpha_i sum_{j in P(i)} ds_ij
//   dw_g[h] = sum_{b,i} dz_i q_i,   db_g[h] = sum_{b,i} dz_i
// Kernels, no atomics (the result does not depend on scheduling):
//   bwd_row_kernel   32 query rows per CTA: each row's softmax and output (online, fp32), D_i,
//                    then dq_i and dz_i; saves lse_i, D_i, the two log2-priors and dz_i per row
//   bwd_key_kernel   32 key rows per CTA: the rows that read them (the index rule read
//                    backwards) accumulate dk_j and dv_j
//   bwd_gate_*       dw_g and db_g, summed over rows in chunks and then over chunks, in a fixed order
// Gradients are fp32 whatever the storage type of the inputs.
#pragma once
#include "common.cuh"
#include "tile_rule.cuh"

namespace pia {

// Per-row values the key kernel and the gate kernel read back (fp32, [B*H*n] each).
struct BwdRowStats {
  float* lse2;  // log2 of the row's softmax denominator (log2 units, as the logits)
  float* D;     // dO_i . out_i
  float* bl2;   // log2(alpha_i): the window prior
  float* bp2;   // log2(1 - alpha_i): the skip prior
  float* dz;    // dLoss / dz_i
};

// ---- tiled kernels -------------------------------------------------------------------------------
// A CTA of 256 threads owns 32 rows (row pass) or 32 keys (key pass); each row or key has 8
// threads, each holding CPT = ceil(d / 8) of its columns, and dot products are reduced over those 8
// lanes.  The other operand streams through shared memory in tiles of kTileKeys rows, chosen by the
// forward's own tile walk (TileWalk: the key tiles a row block reads) or its transpose (ReaderWalk:
// the row tiles that read a key block), and masked by the forward's row_tile_mask -- the same index
// sets as the forward, by construction.  Each warp (4 rows or keys) loops over the union of its
// members' active columns, so every lane takes part in every shuffle.
constexpr int kBwdThreads = 256;
constexpr int kBwdTPR = 8;                       // threads per row / key
constexpr int kBwdRows = kBwdThreads / kBwdTPR;  // rows (or keys) per CTA

// Stage rows [r0, r0 + kTileKeys) of a [n, d] matrix into shared memory (zeros past n).
template <typename T>
__device__ __forceinline__ void stage_tile(T* dst, const T* src, long long r0, long long n, int d) {
  const int vec = 16 / (int)sizeof(T);  // elements per 16-byte chunk
  const int per_row = d / vec;
  for (int idx = threadIdx.x; idx < kTileKeys * per_row; idx += blockDim.x) {
    const int r = idx / per_row, c = (idx % per_row) * vec;
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (r0 + r < n) u = *reinterpret_cast<const uint4*>(src + (r0 + r) * d + c);
    *reinterpret_cast<uint4*>(dst + r * d + c) = u;
  }
}

// The 64 columns of the key tile at j0 that row i reads, as two 32-bit words.
__device__ __forceinline__ void row_tile_bits(long long i, long long j0, int kwin, int pi, int S, int m0, double rpi,
                                              bool bidir, long long n, uint32_t& w0, uint32_t& w1) {
  int lo, hi;
  uint32_t sk[kTileKeys / 32];
  row_tile_mask(i, j0, kwin, pi, S, m0, lo, hi, sk, 0, rpi, bidir, n);
  w0 = window_bits(lo, hi) | sk[0];
  w1 = window_bits(lo - 32, hi - 32) | sk[1];
}

// The CPT columns c0 .. c0 + CPT - 1 of a row in shared memory as fp32, zero past d: 16-byte loads
// when the whole chunk lies in the row (row starts and c0 are 16-byte aligned: d * sizeof(T) is a
// multiple of 16, and so is CPT * sizeof(T)).
template <typename T, int CPT>
__device__ __forceinline__ void load_cols(const T* rowp, int c0, int d, float* f) {
  if (c0 + CPT <= d) {
    if constexpr (sizeof(T) == 2) {
#pragma unroll
      for (int u = 0; u < CPT / 8; ++u) bf16x8_to_f32(*reinterpret_cast<const uint4*>(rowp + c0 + 8 * u), f + 8 * u);
    } else {
#pragma unroll
      for (int u = 0; u < CPT / 4; ++u) {
        const float4 x = *reinterpret_cast<const float4*>(rowp + c0 + 4 * u);
        f[4 * u] = x.x;
        f[4 * u + 1] = x.y;
        f[4 * u + 2] = x.z;
        f[4 * u + 3] = x.w;
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < CPT; ++e) f[e] = c0 + e < d ? to_f32(rowp[c0 + e]) : 0.f;
  }
}
// sum of a[e] * b[e] over the chunk, in packed pairs with two independent accumulators
template <int CPT>
__device__ __forceinline__ float dot_cols(const float* a, const float* b) {
  static_assert(CPT % 4 == 0, "pairs of pairs");
  unsigned long long s0 = 0ull, s1 = 0ull;
#pragma unroll
  for (int e = 0; e < CPT; e += 4) {
    s0 = f2fma(f2pack(a[e], a[e + 1]), f2pack(b[e], b[e + 1]), s0);
    s1 = f2fma(f2pack(a[e + 2], a[e + 3]), f2pack(b[e + 2], b[e + 3]), s1);
  }
  float x, y;
  f2unpack(f2add(s0, s1), x, y);
  return x + y;
}
// acc[e] += s * b[e] over the chunk, in packed pairs
template <int CPT>
__device__ __forceinline__ void axpy_cols(float s, const float* b, float* acc) {
  const unsigned long long s2 = f2pack(s, s);
#pragma unroll
  for (int e = 0; e < CPT; e += 2) f2unpack(f2fma(s2, f2pack(b[e], b[e + 1]), f2pack(acc[e], acc[e + 1])), acc[e], acc[e + 1]);
}
__device__ __forceinline__ float sum8(float x) {  // over the 8 lanes of a row group (all lanes call)
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  return x;
}

// 256-thread CTAs an SM: three for d <= 64 (at most 85 registers a thread), two for d <= 128 (128
// registers); d <= 256 keeps the compiler's choice.
template <int CPT> constexpr int kBwdMinBlocks = CPT <= 8 ? 3 : (CPT <= 16 ? 2 : 1);

template <typename T, int CPT>
__global__ void __launch_bounds__(kBwdThreads, kBwdMinBlocks<CPT>) bwd_row_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                              const T* __restrict__ v, const float* __restrict__ w_g,
                                                              const float* __restrict__ b_g,
                                                              const T* __restrict__ dout, float* __restrict__ dq,
                                                              BwdRowStats st, int H, int n, int d, int kwin, int pi,
                                                              int S, float scale_log2, bool bidir) {
  extern __shared__ __align__(16) uint8_t bwd_smem[];
  T* ks = reinterpret_cast<T*>(bwd_smem);
  T* vs = ks + kTileKeys * d;
  const int tid = threadIdx.x, part = tid & (kBwdTPR - 1), c0 = part * CPT;
  const long long bh = blockIdx.y;
  const int h = (int)(bh % H);
  const long long i0 = (long long)blockIdx.x * kBwdRows, i = i0 + tid / kBwdTPR;
  const bool valid = i < n;
  const long long row = bh * (long long)n + (valid ? i : 0);
  const T* kb = k + bh * (long long)n * d;
  const T* vb = v + bh * (long long)n * d;
  float qr[CPT], gr[CPT], acc[CPT];
#pragma unroll
  for (int e = 0; e < CPT; ++e) {
    const bool in = valid && c0 + e < d;
    qr[e] = in ? to_f32(q[row * d + c0 + e]) : 0.f;
    gr[e] = in ? to_f32(dout[row * d + c0 + e]) : 0.f;
    acc[e] = 0.f;
  }
  float zp = 0.f;
#pragma unroll
  for (int e = 0; e < CPT; ++e)
    if (c0 + e < d) zp = fmaf(qr[e], w_g[(long long)h * d + c0 + e], zp);
  const float z = sum8(zp) + b_g[h];
  const float alpha = 1.f / (1.f + expf(-z));
  const float bl2 = log_sigmoid(z) * kLog2e, bp2 = log_sigmoid(-z) * kLog2e;
  const int m0 = first_skip_m(kwin, pi);
  TileWalk walk;
  walk.init(i0, n, kBwdRows, kwin, pi, S, bidir);

  // the warp walks the columns some of its rows read; each row keeps the ones it reads
  auto tile_cols = [&](long long j0, uint32_t& w0, uint32_t& w1, uint32_t& u0, uint32_t& u1) {
    w0 = w1 = 0u;
    if (valid) row_tile_bits(i, j0, kwin, pi, S, m0, walk.rpi, bidir, n, w0, w1);
    u0 = __reduce_or_sync(0xffffffffu, w0);
    u1 = __reduce_or_sync(0xffffffffu, w1);
  };
  auto is_win = [&](long long j0, int c) {  // a key the row reads is a window key iff |i - j| <= k
    const long long dj = i - (j0 + c);
    return dj <= kwin && dj >= -kwin;
  };

  // the rows' forward: one online softmax over the union, out_i in acc
  float m = -INFINITY, l = 0.f;
  for (int t = walk.next(0); t >= 0; t = walk.next(t + 1)) {
    const long long j0 = (long long)t * kTileKeys;
    __syncthreads();
    stage_tile(ks, kb, j0, n, d);
    stage_tile(vs, vb, j0, n, d);
    __syncthreads();
    uint32_t w0, w1, u0, u1;
    tile_cols(j0, w0, w1, u0, u1);
    for (int half = 0; half < 2; ++half) {
      uint32_t un = half ? u1 : u0;
      const uint32_t mine = half ? w1 : w0;
      while (un) {
        const int b = __ffs(un) - 1;
        un &= un - 1;
        const int c = 32 * half + b;
        float kc[CPT];
        load_cols<T, CPT>(ks + c * d, c0, d, kc);
        const float s = fmaf(sum8(dot_cols<CPT>(qr, kc)), scale_log2, is_win(j0, c) ? bl2 : bp2);
        if ((mine >> b) & 1u) {
          const float mn = fmaxf(m, s);
          const float corr = ex2(m - mn), p = ex2(s - mn);
          l = fmaf(l, corr, p);
          float vc[CPT];
          load_cols<T, CPT>(vs + c * d, c0, d, vc);
          const unsigned long long c2 = f2pack(corr, corr), p2 = f2pack(p, p);
#pragma unroll
          for (int e = 0; e < CPT; e += 2)
            f2unpack(f2fma(f2pack(acc[e], acc[e + 1]), c2, f2mul(p2, f2pack(vc[e], vc[e + 1]))), acc[e], acc[e + 1]);
          m = mn;
        }
      }
    }
  }
  const float lse2 = valid ? m + log2f(l) : 0.f, inv = valid ? 1.f / l : 0.f;
  float Dp = 0.f;
#pragma unroll
  for (int e = 0; e < CPT; ++e) Dp = fmaf(gr[e], acc[e] * inv, Dp);
  const float D = sum8(Dp);

  // the rows' backward
  float dqa[CPT];
#pragma unroll
  for (int e = 0; e < CPT; ++e) dqa[e] = 0.f;
  float dz = 0.f;
  for (int t = walk.next(0); t >= 0; t = walk.next(t + 1)) {
    const long long j0 = (long long)t * kTileKeys;
    __syncthreads();
    stage_tile(ks, kb, j0, n, d);
    stage_tile(vs, vb, j0, n, d);
    __syncthreads();
    uint32_t w0, w1, u0, u1;
    tile_cols(j0, w0, w1, u0, u1);
    for (int half = 0; half < 2; ++half) {
      uint32_t un = half ? u1 : u0;
      const uint32_t mine = half ? w1 : w0;
      while (un) {
        const int b = __ffs(un) - 1;
        un &= un - 1;
        const int c = 32 * half + b;
        const bool win = is_win(j0, c);
        float kc[CPT], vc[CPT];
        load_cols<T, CPT>(ks + c * d, c0, d, kc);
        load_cols<T, CPT>(vs + c * d, c0, d, vc);
        const float s = fmaf(sum8(dot_cols<CPT>(qr, kc)), scale_log2, win ? bl2 : bp2);
        const float dp = sum8(dot_cols<CPT>(gr, vc));
        if ((mine >> b) & 1u) {
          const float ds = ex2(s - lse2) * (dp - D);
          dz += win ? (1.f - alpha) * ds : -alpha * ds;
          axpy_cols<CPT>(ds, kc, dqa);
        }
      }
    }
  }
  const float tau = scale_log2 / kLog2e;
  if (valid) {
#pragma unroll
    for (int e = 0; e < CPT; ++e)
      if (c0 + e < d) dq[row * d + c0 + e] = fmaf(tau, dqa[e], dz * w_g[(long long)h * d + c0 + e]);
    if (part == 0) {
      st.lse2[row] = lse2;
      st.D[row] = D;
      st.bl2[row] = bl2;
      st.bp2[row] = bp2;
      st.dz[row] = dz;
    }
  }
}

template <typename T, int CPT>
__global__ void __launch_bounds__(kBwdThreads, kBwdMinBlocks<CPT>) bwd_key_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                              const T* __restrict__ v, const T* __restrict__ dout,
                                                              BwdRowStats st, float* __restrict__ dk,
                                                              float* __restrict__ dv, int H, int n, int d, int kwin,
                                                              int pi, int S, float scale_log2, bool bidir) {
  extern __shared__ __align__(16) uint8_t bwd_smem[];
  T* qs = reinterpret_cast<T*>(bwd_smem);
  T* gs = qs + kTileKeys * d;
  float* rstat = reinterpret_cast<float*>(gs + kTileKeys * d);  // [4][kTileKeys]: lse2, D, bl2, bp2
  uint32_t* rbits = reinterpret_cast<uint32_t*>(rstat + 4 * kTileKeys);  // [kTileKeys]: this block's 32 keys
  const int tid = threadIdx.x, part = tid & (kBwdTPR - 1), c0 = part * CPT;
  const long long bh = blockIdx.y;
  (void)H;
  const long long j0 = (long long)blockIdx.x * kBwdRows, j = j0 + tid / kBwdTPR;
  const bool valid = j < n;
  const long long key = bh * (long long)n + (valid ? j : 0);
  const long long rbase = bh * (long long)n;
  const long long J0 = j0 / kTileKeys * kTileKeys;  // the 64-key tile holding this block's keys
  const int off = (int)(j0 - J0);                    // 0 or 32
  const int kc = (int)(j - j0);                       // this key's bit in the block's word
  float kr[CPT], vr[CPT], dka[CPT], dva[CPT];
#pragma unroll
  for (int e = 0; e < CPT; ++e) {
    const bool in = valid && c0 + e < d;
    kr[e] = in ? to_f32(k[key * d + c0 + e]) : 0.f;
    vr[e] = in ? to_f32(v[key * d + c0 + e]) : 0.f;
    dka[e] = dva[e] = 0.f;
  }
  const int m0 = first_skip_m(kwin, pi);
  ReaderWalk walk;
  walk.init(j0, n, kBwdRows, kwin, pi, S, bidir);
  const double rpi = 1.0 / (double)pi;
  const int wkeys = (tid >> 5) * 4;  // this warp's 4 keys: bits wkeys .. wkeys + 3 of a row's word
  for (int t = walk.next(0); t >= 0; t = walk.next(t + 1)) {
    const long long r0 = (long long)t * kTileKeys;
    __syncthreads();
    stage_tile(qs, q + rbase * d, r0, n, d);
    stage_tile(gs, dout + rbase * d, r0, n, d);
    if (tid < kTileKeys) {
      const long long i = r0 + tid;
      uint32_t w = 0u;
      float a = 0.f, b = 0.f, c = 0.f, e = 0.f;
      if (i < n) {
        uint32_t w0, w1;
        row_tile_bits(i, J0, kwin, pi, S, m0, rpi, bidir, n, w0, w1);
        w = off ? w1 : w0;
        a = st.lse2[rbase + i];
        b = st.D[rbase + i];
        c = st.bl2[rbase + i];
        e = st.bp2[rbase + i];
      }
      rbits[tid] = w;
      rstat[tid] = a;
      rstat[kTileKeys + tid] = b;
      rstat[2 * kTileKeys + tid] = c;
      rstat[3 * kTileKeys + tid] = e;
    }
    __syncthreads();
    for (int r = 0; r < kTileKeys; ++r) {
      const uint32_t w = rbits[r];
      if (((w >> wkeys) & 0xFu) == 0u) continue;  // no key of this warp is read by row r (warp-uniform)
      const long long i = r0 + r;
      const long long dj = i - j;
      const bool win = dj <= kwin && dj >= -kwin;
      float qc[CPT], gc[CPT];
      load_cols<T, CPT>(qs + r * d, c0, d, qc);
      load_cols<T, CPT>(gs + r * d, c0, d, gc);
      const float s = fmaf(sum8(dot_cols<CPT>(kr, qc)), scale_log2, win ? rstat[2 * kTileKeys + r] : rstat[3 * kTileKeys + r]);
      const float dp = sum8(dot_cols<CPT>(vr, gc));
      if (valid && ((w >> kc) & 1u)) {
        const float p = ex2(s - rstat[r]);
        const float ds = p * (dp - rstat[kTileKeys + r]);
        axpy_cols<CPT>(p, gc, dva);
        axpy_cols<CPT>(ds, qc, dka);
      }
    }
  }
  const float tau = scale_log2 / kLog2e;
  if (valid) {
#pragma unroll
    for (int e = 0; e < CPT; ++e) {
      if (c0 + e < d) {
        dk[key * d + c0 + e] = tau * dka[e];
        dv[key * d + c0 + e] = dva[e];
      }
    }
  }
}

// dynamic shared memory of the tiled kernels
inline size_t bwd_row_smem(int d, size_t esz) { return 2 * (size_t)kTileKeys * d * esz; }
inline size_t bwd_key_smem(int d, size_t esz) { return 2 * (size_t)kTileKeys * d * esz + 5 * kTileKeys * 4; }

// dw_g[h][c] = sum over (b, i) of dz * q[c], db_g[h] = sum of dz, in two stages with a fixed order:
// bwd_gate_partial_kernel sums chunks of kGateRows rows of one head (one block per (chunk, head),
// one thread per column), bwd_gate_final_kernel adds the chunks in a fixed order.
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

// Grid (H, ceil(d / 32)), 1024 threads: 32 columns x 32 chunk groups.  Thread (g, c) adds the
// chunks g, g + 32, ... of column c into four interleaved sums (independent loads in flight), and a
// fixed tree then adds the 32 group sums; the blocks of column group 0 also add part_b the same way
// over all 1024 threads.  The order is fixed for a given nchunks: the result does not depend on
// scheduling.
__global__ void __launch_bounds__(1024) bwd_gate_final_kernel(const float* __restrict__ part_w,
                                                              const float* __restrict__ part_b,
                                                              float* __restrict__ dw_g, float* __restrict__ db_g,
                                                              int nchunks, int d) {
  __shared__ float red[32][33];
  __shared__ float red_b[1024];
  const int h = blockIdx.x, tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int c = blockIdx.y * 32 + tx;
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  if (c < d) {
    const float* pw = part_w + (long long)h * nchunks * d + c;
    int k = ty;
    for (; k + 96 < nchunks; k += 128) {
      a0 += pw[(long long)k * d];
      a1 += pw[(long long)(k + 32) * d];
      a2 += pw[(long long)(k + 64) * d];
      a3 += pw[(long long)(k + 96) * d];
    }
    for (; k < nchunks; k += 32) a0 += pw[(long long)k * d];
  }
  red[ty][tx] = (a0 + a1) + (a2 + a3);
  const bool do_b = blockIdx.y == 0;
  if (do_b) {
    const float* pb = part_b + (long long)h * nchunks;
    float b0 = 0.f, b1 = 0.f;
    int k = threadIdx.x;
    for (; k + 1024 < nchunks; k += 2048) {
      b0 += pb[k];
      b1 += pb[k + 1024];
    }
    if (k < nchunks) b0 += pb[k];
    red_b[threadIdx.x] = b0 + b1;
  }
  __syncthreads();
  for (int st = 16; st > 0; st >>= 1) {
    if (ty < st) red[ty][tx] += red[ty + st][tx];
    __syncthreads();
  }
  if (ty == 0 && c < d) dw_g[(long long)h * d + c] = red[0][tx];
  if (do_b) {  // uniform over the block
    for (int st = 512; st > 0; st >>= 1) {
      if ((int)threadIdx.x < st) red_b[threadIdx.x] += red_b[threadIdx.x + st];
      __syncthreads();
    }
    if (threadIdx.x == 0) db_g[h] = red_b[0];
  }
}

}  // namespace pia
