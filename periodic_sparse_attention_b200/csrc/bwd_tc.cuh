// bwd_tc.cuh -- the backward's dq pass and dk/dv pass on Blackwell tensor cores (tcgen05 + TMEM +
// TMA), bf16, head size 64 or 128.  Each runs in the sequence view (window and skips in one
// sweep, or the window alone) or in the residue-class view of the split path (the skips alone).
//
// The dq pass:
// One CTA per (query tile of 128 rows, b, h), walking the key tiles of the forward (the same
// TileCursor over the same index rule).  Per 64-key tile:
//   MMA warp            S = Q K^T and dP = dO V^T (fp32 in TMEM), then, once the softmax warps
//                       have written dS, dQ += dS K (fp32 in TMEM; dS from TMEM, K N-major)
//   softmax warpgroup   one thread per query row: p = 2^(s tau log2e + prior - lse2) on the keys
//                       the index rule gives (0 elsewhere), ds = p (dp - D), written in bf16 over
//                       the S columns already read; the row's dz = (1 - alpha) sum_window ds -
//                       alpha sum_skip ds (the gate's gradient through the two log-priors)
//   TMA producer warp   Q and dO tiles once, then K and V tiles into a ring of NSTAGE stages
// lse and D = dO . out of every row come from the forward pass (its epilogue forms D from the
// fp32 output rows).  The epilogue writes dq = tau dQ + dz w_g (fp32) and the rows' dz, which the
// gate sums read.
//
// TMEM: NBUF pairs of S (64 columns) and dP (64), then dQ (D columns).  D = 64 (two CTAs an SM):
// one pair and one softmax warpgroup, the next tile's Q K^T waits for this tile's dS K (it reads
// dS over the S columns).  D = 128 (one CTA an SM): two pairs and two softmax warpgroups taking
// the tiles in turn (even tiles pair 0, odd tiles pair 1), the MMA warp issuing tile j + 1's
// Q K^T before tile j's dS K, so one group's softmax runs while the other's MMAs do; the groups
// add their rows' dz sums in a fixed order at the end and share the epilogue's columns.  The
// epilogues wait on the drain barrier, committed after the MMA warp's last issue.  Every wait is
// bounded as in the forward kernel; a wait that gives up sets the error word and the abort flag,
// and every role leaves, drains its own asynchronous work and the CTA frees its TMEM.
#pragma once
#include "fwd_tc.cuh"

namespace pia {
namespace tcb {
using tc::BM;
using tc::BN;
// Depth of the ring of streamed tiles (K and V in the dq pass, Q and dO in the dk/dv pass): a
// stage is held until the tile's last MMA has completed, and the load into it must land before
// the tile NSTAGE later is needed.
constexpr int NSTAGE = 4;

template <int D>
struct BSmem {
  static constexpr int kCtas = D == 64 ? 2 : 1;         // shared memory: 97 KB (D = 64) or 194 KB
  static constexpr int kNbuf = D == 64 ? 1 : 2;         // S/dP pairs in TMEM = softmax warpgroups
  static constexpr int kThreads = 64 + 128 * kNbuf;
  static constexpr int kTileBytes = BM * D * 2;          // the Q tile, the dO tile
  static constexpr int kKVBytes = BN * D * 2;            // one K or V tile
  static constexpr int kQ = 0;
  static constexpr int kG = kQ + kTileBytes;
  static constexpr int kK = kG + kTileBytes;
  static constexpr int kV = kK + NSTAGE * kKVBytes;
  static constexpr int kBar = kV + NSTAGE * kKVBytes;
  // barriers: qg_full, k_full[NSTAGE], k_empty[NSTAGE], v_full[NSTAGE], v_empty[NSTAGE],
  // s_full[kNbuf], ds_full[kNbuf], dq_done[kNbuf], drain
  static constexpr int kNumBars = 1 + 4 * NSTAGE + 3 * kNbuf + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;      // tmem base (4 B), abort flag (4 B)
  static constexpr int kWg = (kMisc + 8 + 15) / 16 * 16; // w_g[h], D floats
  static constexpr int kDz = kWg + D * 4;                // the rows' dz, then the gate partials (BM floats each)
  static constexpr int kRed = kDz + BM * 4;
  static constexpr int kComb = kRed + BM * 4;            // each warpgroup's dz sums (window, skip) per row
  static constexpr int kTotal = kComb + kNbuf * 2 * BM * 4;
  static constexpr int kAlloc = kTotal + 1024 - 128;
  static constexpr int kTmemCols = kNbuf == 1 ? 256 : 512;
  static_assert(2 * BN * kNbuf + D <= kTmemCols && kTmemCols * kCtas <= 512, "TMEM columns");
  static_assert(kQ % 1024 == 0 && kG % 1024 == 0 && kK % 1024 == 0 && kV % 1024 == 0 && kKVBytes % 1024 == 0,
                "128-byte-swizzled tiles sit on 1 KB");
  static_assert(kBar % 8 == 0 && kWg % 16 == 0, "mbarriers on 8 bytes, the w_g staging on 16");
  static_assert(kAlloc <= 228 * 1024 / kCtas - 1024, "shared memory of the CTAs on one SM");
};

struct BParams {
  const float* w_g;
  const float* b_g;
  const float* lse;   // [B*H, n] the forward's lse (natural log)
  const float* Dr;    // [B*H, n] dO . out
  float* dq;          // [B*H, n, D]
  float* dz;          // [B*H, n] dLoss / dz_i, for the gate
  float* part_w;      // [H, B * tiles, D] this CTA's sum of dz_i q_i over its rows, in chunk b * tiles + tile
  float* part_b;      // [H, B * tiles]    and of dz_i
  int H, n, kwin, pi, S;
  float scale_log2;
  int bidir;
  int acc;            // add to the dq and dz that the residue pass wrote (the split backward)
};

// RES = 0: the sequence view, the rule's window and skips (S = 0: the window alone).  RES = 1: the
// skips alone, in the residue-class view of the forward's split path: the CTA's rows are rows
// t*pi + res of the sequence, their skip keys the band t - S .. t - m0 of the same class (all with
// the skip prior).  The residue pass runs first and writes its dq and dz; the window pass then
// runs with acc set, adds to both, and takes the gate's partial sums over the whole dz.
template <int D, int RES>
__global__ void __launch_bounds__(BSmem<D>::kThreads, BSmem<D>::kCtas) bwd_dq_kernel(const __grid_constant__ CUtensorMap tmq,
                                                                       const __grid_constant__ CUtensorMap tmg,
                                                                       const __grid_constant__ CUtensorMap tmk,
                                                                       const __grid_constant__ CUtensorMap tmv,
                                                                       BParams prm) {
  using namespace tc;
  using L = BSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const sbase = smem_raw + (base - raw);
  if (base - raw + L::kTotal > (uint32_t)L::kAlloc) {
    if (threadIdx.x == 0) raise_error(kErrInternal);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int h = bh % prm.H;
  const int res = RES ? (int)(blockIdx.x % prm.pi) : 0;
  const long long q0 = RES ? (long long)(blockIdx.x / prm.pi) * BM : (long long)blockIdx.x * BM;
  const long long T = RES ? prm.n / prm.pi : prm.n;  // rows of the view
  const uint32_t sQ = base + L::kQ, sG = base + L::kG, sK = base + L::kK, sV = base + L::kV;
  const uint32_t bar0 = base + L::kBar;
  const uint32_t bar_qg = bar0;
  auto bar_kfull = [&](int s) { return bar0 + 8u * (1 + s); };
  auto bar_kempty = [&](int s) { return bar0 + 8u * (1 + NSTAGE + s); };
  auto bar_vfull = [&](int s) { return bar0 + 8u * (1 + 2 * NSTAGE + s); };
  auto bar_vempty = [&](int s) { return bar0 + 8u * (1 + 3 * NSTAGE + s); };
  constexpr int NBUF = L::kNbuf;
  auto bar_sfull = [&](int b) { return bar0 + 8u * (1 + 4 * NSTAGE + b); };
  auto bar_dsfull = [&](int b) { return bar0 + 8u * (1 + 4 * NSTAGE + NBUF + b); };
  auto bar_dqdone = [&](int b) { return bar0 + 8u * (1 + 4 * NSTAGE + 2 * NBUF + b); };
  const uint32_t bar_drain = bar0 + 8u * (1 + 4 * NSTAGE + 3 * NBUF);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(sbase + L::kMisc);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(sbase + L::kMisc + 4);

  // Q and dO first: their latency heads every CTA's critical path
  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmq) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmg) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmk) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmv) : "memory");
    mbar_init(bar_qg, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_expect_tx(bar_qg, 2 * L::kTileBytes);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      if (RES) {
        tma_load_4d(sQ + c * BM * 128, &tmq, bar_qg, c * 64, res, (int)q0, bh);
        tma_load_4d(sG + c * BM * 128, &tmg, bar_qg, c * 64, res, (int)q0, bh);
      } else {
        tma_load_3d(sQ + c * BM * 128, &tmq, bar_qg, c * 64, (int)q0, bh);
        tma_load_3d(sG + c * BM * 128, &tmg, bar_qg, c * 64, (int)q0, bh);
      }
    }
  }
  const int m0 = first_skip_m(prm.kwin, prm.pi);
  TileWalk walk;
  if (RES) {  // keys of view row t: t - S .. t - m0
    walk.init_residue(q0, T, BM, prm.S, m0);
  } else {
    walk.init(q0, prm.n, BM, prm.kwin, prm.pi, prm.S, prm.bidir != 0);
  }
  TileCursor cur;
  cur.init(walk);
  int t_first = -1;
  auto load_kv = [&](uint32_t dst, const CUtensorMap* map, uint32_t bar, long long r0) {
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      if (RES)
        tma_load_4d(dst + c * BN * 128, map, bar, c * 64, res, (int)r0, bh);
      else
        tma_load_3d(dst + c * BN * 128, map, bar, c * 64, (int)r0, bh);
    }
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(bar_kfull(s), 1);
      mbar_init(bar_kempty(s), 1);
      mbar_init(bar_vfull(s), 1);
      mbar_init(bar_vempty(s), 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(bar_sfull(b), 1);
      mbar_init(bar_dsfull(b), BM);
      mbar_init(bar_dqdone(b), 1);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    t_first = cur.next();
    if (t_first >= 0) {
      mbar_expect_tx(bar_kfull(0), L::kKVBytes);
      load_kv(sK, &tmk, bar_kfull(0), (long long)t_first * BN);
      mbar_expect_tx(bar_vfull(0), L::kKVBytes);
      load_kv(sV, &tmv, bar_vfull(0), (long long)t_first * BN);
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "n"(L::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // pair b: S at b * 128, dP at b * 128 + 64; dQ after the pairs
  const uint32_t tQ = tmem + 2 * BN * NBUF;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      constexpr uint32_t kKV = L::kKVBytes;
      int nk = t_first >= 0 ? 1 : 0, nv = nk;
      for (int t = cur.next(); t >= 0; t = cur.next()) {
        const int s = nk % NSTAGE, use = nk / NSTAGE;
        if (use > 0 && !mbar_wait(bar_kempty(s), (use - 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_kfull(s), kKV);
        load_kv(sK + s * kKV, &tmk, bar_kfull(s), (long long)t * BN);
        ++nk;
        if (use > 0 && !mbar_wait(bar_vempty(s), (use - 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_vfull(s), kKV);
        load_kv(sV + s * kKV, &tmv, bar_vfull(s), (long long)t * BN);
        ++nv;
      }
      if (*abort_flag) {  // let the loads already in flight land before the CTA can exit
        volatile int never = 0;
        mbar_wait(bar_qg, 0, &never);
        for (int u = nk > NSTAGE ? nk - NSTAGE : 0; u < nk; ++u)
          mbar_wait(bar_kfull(u % NSTAGE), (u / NSTAGE) & 1, &never);
        for (int u = nv > NSTAGE ? nv - NSTAGE : 0; u < nv; ++u)
          mbar_wait(bar_vfull(u % NSTAGE), (u / NSTAGE) & 1, &never);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kKV = L::kKVBytes;
      constexpr uint32_t idesc_s = idesc_bf16(BM, BN, 0);  // S, dP: B (K, V) K-major
      constexpr uint32_t idesc_q = idesc_bf16(BM, D, 1);   // dQ: B (K) N-major
      bool okw = mbar_wait(bar_qg, 0, abort_flag);
      tc_fence_after();
      // S = Q K^T, dP = dO V^T of tile j into pair j % NBUF
      auto issue_s = [&](int j) -> bool {
        const int s = j % NSTAGE, b = j % NBUF;
        if (!mbar_wait(bar_kfull(s), (j / NSTAGE) & 1, abort_flag)) return false;
        if (!mbar_wait(bar_vfull(s), (j / NSTAGE) & 1, abort_flag)) return false;
        // the dS K of tile j - NBUF read dS over the S columns this Q K^T overwrites
        if (j >= NBUF && !mbar_wait(bar_dqdone(b), ((j - NBUF) / NBUF) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t tS = tmem + b * 2 * BN, tP = tS + BN;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t in = (kk & 3) * 32;
          tc_mma(tS, sw128_desc(sQ + (kk >> 2) * (BM * 128) + in, 16, 1024),
                 sw128_desc(sK + s * kKV + (kk >> 2) * (BN * 128) + in, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t in = (kk & 3) * 32;
          tc_mma(tP, sw128_desc(sG + (kk >> 2) * (BM * 128) + in, 16, 1024),
                 sw128_desc(sV + s * kKV + (kk >> 2) * (BN * 128) + in, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar_sfull(b));
        tc_commit(bar_vempty(s));  // V was read by dO V^T only
        return true;
      };
      // dQ += dS K of tile j: K = BN keys, 16 per instruction; dS packed two per column over S
      auto issue_dq = [&](int j) -> bool {
        const int s = j % NSTAGE, b = j % NBUF;
        if (!mbar_wait(bar_dsfull(b), (j / NBUF) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t tS = tmem + b * 2 * BN;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t acol = 16 * (kk >> 1) + 8 * (kk & 1);
          tc_mma_ts(tQ, tS + acol, sw128_desc(sK + s * kKV + kk * 16 * 128, BN * 128, 1024), idesc_q,
                    (j == 0 && kk == 0) ? 0u : 1u);
        }
        tc_commit(bar_dqdone(b));
        tc_commit(bar_kempty(s));
        return true;
      };
      // one pair: dS K of tile j - 1, then Q K^T of tile j; two pairs: Q K^T of tile j first
      int j = 0;
      for (int t = cur.next(); okw; t = cur.next(), ++j) {
        const bool have = t >= 0;
        if (NBUF == 1 && j > 0 && !issue_dq(j - 1)) break;
        if (have && !issue_s(j)) break;
        if (NBUF == 2 && j > 0 && !issue_dq(j - 1)) break;
        if (!have) break;
      }
      tc_commit(bar_drain);
      volatile int never = 0;
      mbar_wait(bar_drain, 0, &never);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    const int wg = (warp - 2) >> 2;  // takes the tiles j with j % NBUF == wg, in pair wg
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const long long qi = q0 + r;                       // row of the view
    const long long i = RES ? qi * prm.pi + res : qi;  // row of the sequence
    const bool row_ok = qi < T;
    const long long orow = (long long)bh * prm.n + (row_ok ? i : 0);
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float lse2 = row_ok ? prm.lse[orow] * kLog2e : 0.f;
    const float Drow = row_ok ? prm.Dr[orow] : 0.f;
    // RES: the band of view columns qi - S .. qi - m0 (every one a skip key)
    const long long w_lo = RES ? (qi - prm.S > 0 ? qi - prm.S : 0) : (i - prm.kwin > 0 ? i - prm.kwin : 0);
    const long long w_hi = RES ? qi - m0 : (prm.bidir ? (i + prm.kwin < prm.n - 1 ? i + prm.kwin : prm.n - 1) : i);
    RowSkips rs;
    rs.init(i, prm.pi, RES ? 0 : prm.S, m0, walk.rpi, prm.bidir != 0, prm.n);

    float* const wg_s = reinterpret_cast<float*>(sbase + L::kWg);
    if (threadIdx.x - 64 < D) wg_s[threadIdx.x - 64] = prm.w_g[(long long)h * D + (threadIdx.x - 64)];
    float z = prm.b_g[h];
    asm volatile("bar.sync 2, %0;" ::"r"(128 * NBUF) : "memory");
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar_qg, 0, abort_flag));
    {
      float zp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        const int blk = c >> 3, cc = c & 7;
        const uint4 u = *reinterpret_cast<const uint4*>(sbase + L::kQ + blk * (BM * 128) + r * 128 +
                                                        ((cc ^ (r & 7)) << 4));
        float f[8];
        bf16x8_to_f32(u, f);
        const float4 w0 = reinterpret_cast<const float4*>(wg_s)[2 * c];
        const float4 w1 = reinterpret_cast<const float4*>(wg_s)[2 * c + 1];
        zp[0] = fmaf(f[0], w0.x, zp[0]);
        zp[1] = fmaf(f[1], w0.y, zp[1]);
        zp[2] = fmaf(f[2], w0.z, zp[2]);
        zp[3] = fmaf(f[3], w0.w, zp[3]);
        zp[0] = fmaf(f[4], w1.x, zp[0]);
        zp[1] = fmaf(f[5], w1.y, zp[1]);
        zp[2] = fmaf(f[6], w1.z, zp[2]);
        zp[3] = fmaf(f[7], w1.w, zp[3]);
      }
      z += (zp[0] + zp[1]) + (zp[2] + zp[3]);
    }
    const float ls_a = log_sigmoid_fast(z), ls_b = log_sigmoid_fast(-z);
    const float alpha = __expf(ls_a);
    const float bl2 = ls_a * kLog2e, bp2 = ls_b * kLog2e;
    const float bl_m = (RES ? bp2 : bl2) - lse2, bp_m = bp2 - lse2;  // RES: the band is skip keys
    const float NEG_INF = -INFINITY;
    float dzw = 0.f, dzs = 0.f;  // sums of ds over window keys and over skip keys

    const uint32_t tS = tmem + wg * 2 * BN, tP = tS + BN;
    int j = 0;
    for (int t = cur.next(); ok && t >= 0; t = cur.next(), ++j) {
      if (j % NBUF != wg) continue;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_sfull(wg), (j / NBUF) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const long long j0 = (long long)t * BN;
      const long long lo64 = w_lo - j0, hi64 = w_hi - j0;
      const int lc_lo = lo64 < 0 ? 0 : (lo64 > BN ? BN : (int)lo64);
      const int lc_hi = hi64 > BN - 1 ? BN - 1 : (hi64 < -1 ? -1 : (int)hi64);
      const uint64_t skw = rs.take(j0);
#pragma unroll 1
      for (int cb = 0; cb < BN / 32; ++cb) {
        const int c0 = cb * 32;
        float x[32], g[32];
        tmem_ld32(tS + lane_off + c0, x);
        tmem_ld32(tP + lane_off + c0, g);
        const uint32_t wm = window_bits(lc_lo - c0, lc_hi - c0);
        const uint32_t skb = (uint32_t)(skw >> c0);
        uint32_t pk[16];
        if ((wm | skb) == 0u) {
#pragma unroll
          for (int w = 0; w < 16; ++w) pk[w] = 0u;
        } else {
          const unsigned long long sc2 = f2pack(prm.scale_log2, prm.scale_log2);
          const unsigned long long nd2 = f2pack(-Drow, -Drow);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const bool w0 = (wm >> e) & 1u, w1 = (wm >> (e + 1)) & 1u;
            const bool s0 = (skb >> e) & 1u, s1 = (skb >> (e + 1)) & 1u;
            const float b0 = w0 ? bl_m : (s0 ? bp_m : NEG_INF);
            const float b1 = w1 ? bl_m : (s1 ? bp_m : NEG_INF);
            float t0, t1;
            f2unpack(f2fma(f2pack(x[e], x[e + 1]), sc2, f2pack(b0, b1)), t0, t1);
            float ds0, ds1;
            f2unpack(f2mul(f2pack(ex2(t0), ex2(t1)), f2add(f2pack(g[e], g[e + 1]), nd2)), ds0, ds1);
            dzw += (w0 ? ds0 : 0.f) + (w1 ? ds1 : 0.f);
            dzs += (s0 ? ds0 : 0.f) + (s1 ? ds1 : 0.f);
            __nv_bfloat162 b2 = __floats2bfloat162_rn(ds0, ds1);
            pk[e >> 1] = *reinterpret_cast<uint32_t*>(&b2);
          }
        }
        __syncwarp();
        tmem_st16(tS + lane_off + 16 * cb, pk);  // over S columns already read
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_dsfull(wg));
    }
    if (NBUF == 2) {  // both groups' sums, added in group order by each group
      float* const comb = reinterpret_cast<float*>(sbase + L::kComb);
      comb[wg * 2 * BM + r] = dzw;
      comb[wg * 2 * BM + BM + r] = dzs;
      asm volatile("bar.sync 3, %0;" ::"r"(128 * NBUF) : "memory");
      dzw = comb[r] + comb[2 * BM + r];
      dzs = comb[BM + r] + comb[3 * BM + r];
    }
    {
      // ---- epilogue: dq = tau dQ + dz w_g (each group its share of the columns), and (group 0)
      // the rows' dz
      if (RES) {  // the band columns were skip keys
        dzs += dzw;
        dzw = 0.f;
      }
      // this pass's dz goes into its dq; the row's whole dz (with the residue pass's part, whose dq
      // already holds its own) into the gate's sums
      const float dz_own = (1.f - alpha) * dzw - alpha * dzs;
      const float dz = !RES && prm.acc && row_ok ? dz_own + prm.dz[orow] : dz_own;
      // every MMA done: the drain barrier, committed once after the MMA warp's last issue (a
      // pair's own barrier could alias: its parity says nothing to a group that skipped phases)
      const bool have_q = __all_sync(0xffffffffu, ok && j > 0 && mbar_wait(bar_drain, 0, abort_flag));
      if (have_q) tc_fence_after();
      const float tau = prm.scale_log2 / kLog2e;
      if (have_q || j == 0) {
        constexpr int kChunks = D / 32 / NBUF;  // 32-column chunks a group
#pragma unroll 1
        for (int c = wg * kChunks; c < (wg + 1) * kChunks; ++c) {
          float4* dst = reinterpret_cast<float4*>(prm.dq + orow * D + c * 32);
          float4 prev[8];  // the residue pass's dq, loaded before the TMEM read to overlap it
          if (!RES && prm.acc && row_ok) {
#pragma unroll
            for (int e = 0; e < 8; ++e) prev[e] = dst[e];
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) prev[e] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
          float o[32];
          if (have_q) {
            tmem_ld32(tQ + lane_off + c * 32, o);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0.f;
          }
          if (row_ok) {
            const float4* wv = reinterpret_cast<const float4*>(wg_s + c * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 w = wv[e], a = prev[e];
              dst[e] = make_float4(a.x + fmaf(tau, o[4 * e], dz_own * w.x), a.y + fmaf(tau, o[4 * e + 1], dz_own * w.y),
                                   a.z + fmaf(tau, o[4 * e + 2], dz_own * w.z),
                                   a.w + fmaf(tau, o[4 * e + 3], dz_own * w.w));
            }
          }
        }
      }
      if (wg == 0 && (have_q || j == 0)) {
        if (row_ok) prm.dz[orow] = dz;
      }
      // The gate's partial sums over this CTA's rows, in a fixed order: dw_g[c] += sum_r dz_r q_rc
      // and db_g += sum_r dz_r.  G = BM / D threads a column, each over BM / G rows of the Q tile
      // (still in shared memory), then the G parts in order.  Group 0 alone.
      if (!RES && wg == 0) {
        float* const dz_s = reinterpret_cast<float*>(sbase + L::kDz);
        float* const red = reinterpret_cast<float*>(sbase + L::kRed);
        dz_s[r] = (have_q || j == 0) && row_ok ? dz : 0.f;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        constexpr int G = BM / D, RPT = BM / G;
        const int c = r % D, g = r / D;
        float acc = 0.f;
#pragma unroll 4
        for (int rr = g * RPT; rr < (g + 1) * RPT; ++rr) {
          const int cc = c & 63;
          const uint32_t off = (c >> 6) * (BM * 128) + rr * 128 + ((((cc >> 3) ^ (rr & 7))) << 4) + (cc & 7) * 2;
          const float qv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sbase + L::kQ + off));
          acc = fmaf(dz_s[rr], qv, acc);
        }
        red[r] = acc;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const long long chunk = (long long)(bh / prm.H) * gridDim.x + blockIdx.x;
        const long long nchunks = (long long)(gridDim.y / prm.H) * gridDim.x;
        if (r < D) {
          float sw = 0.f;
#pragma unroll
          for (int gg = 0; gg < G; ++gg) sw += red[gg * D + r];
          prm.part_w[((long long)h * nchunks + chunk) * D + r] = sw;
        }
        if (r == 0) {
          float sb = 0.f;
          for (int rr = 0; rr < BM; ++rr) sb += dz_s[rr];
          prm.part_b[(long long)h * nchunks + chunk] = sb;
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(L::kTmemCols) : "memory");
  }
}

// ---- the dk/dv pass: the forward's roles swapped ---------------------------------------------
// One CTA per (block of 128 keys, b, h), walking the 64-row tiles that read its keys
// (ReaderWalk).  Per row tile:
//   MMA warp            S^T = K Q^T and dP^T = V dO^T (128 keys x 64 rows, fp32 in TMEM), then,
//                       once the softmax warps have written P^T and dS^T, dV += P^T dO and
//                       dK += dS^T Q (fp32 in TMEM; P^T, dS^T from TMEM, dO and Q N-major)
//   softmax warpgroup   one thread per key: for each row that reads the key (its window rows, a
//                       range, and its skip rows, KeyReaders) p = 2^(s tau log2e + prior - lse2)
//                       and ds = p (dp - D) from the row's terms (staged in shared memory), P^T
//                       and dS^T in bf16 over the S^T and dP^T columns already read
//   TMA producer warp   K and V tiles once, then Q and dO row tiles into a ring of NSTAGE stages
// The epilogue writes dk = tau dK, dv = dV (fp32).  TMEM: NBUF pairs of S^T (64 columns) and dP^T
// (64), dV and dK after them: D = 64 one pair and one key warpgroup (256 columns, two CTAs an
// SM); D = 128 two pairs and two key warpgroups taking the row tiles in turn, the MMA warp issuing
// tile j + 1's S^T, dP^T before tile j's dV, dK MMAs (512 columns, one CTA an SM); in the
// epilogue warpgroup 0 writes dk and warpgroup 1 dv.
template <int D>
struct KSmem {
  static constexpr int kCtas = D == 64 ? 2 : 1;
  static constexpr int kNbuf = D == 64 ? 1 : 2;          // S^T/dP^T pairs in TMEM = key warpgroups
  static constexpr int kThreads = 64 + 128 * kNbuf;
  static constexpr int kKeyBytes = BM * D * 2;           // the K tile, the V tile (128 keys)
  static constexpr int kRowBytes = BN * D * 2;           // one Q or dO row tile (64 rows)
  static constexpr int kK = 0;
  static constexpr int kV = kK + kKeyBytes;
  static constexpr int kQ = kV + kKeyBytes;
  static constexpr int kG = kQ + NSTAGE * kRowBytes;
  // 2 buffers a key warpgroup x 64 rows x (lse2, D, bl2, bp2)
  static constexpr int kStat = kG + NSTAGE * kRowBytes;
  static constexpr int kBar = kStat + 2 * kNbuf * BN * 16;
  // barriers: kv_full, q_full[NSTAGE], q_empty[NSTAGE], g_full[NSTAGE], g_empty[NSTAGE],
  // s_full[kNbuf], p_full[kNbuf], kv_done[kNbuf], drain
  static constexpr int kNumBars = 1 + 4 * NSTAGE + 3 * kNbuf + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kTotal = kMisc + 8;
  static constexpr int kAlloc = kTotal + 1024 - 128;
  static constexpr int kTmemCols = D == 64 ? 256 : 512;
  static_assert(2 * BN * kNbuf + 2 * D <= kTmemCols && kTmemCols * kCtas <= 512, "TMEM columns");
  static_assert(kK % 1024 == 0 && kV % 1024 == 0 && kQ % 1024 == 0 && kG % 1024 == 0 && kRowBytes % 1024 == 0,
                "128-byte-swizzled tiles sit on 1 KB");
  static_assert(kStat % 16 == 0 && kBar % 8 == 0, "row terms on 16 bytes, mbarriers on 8");
  static_assert(kAlloc <= 228 * 1024 / kCtas - 1024, "shared memory of the CTAs on one SM");
};

struct KParams {
  const float* lse2;  // [B*H, n] the rows' terms, written by the forward that precedes the backward
  const float* Dr;
  const float* bl2;
  const float* bp2;
  float* dk;          // [B*H, n, D]
  float* dv;
  int n, kwin, pi, S;
  float scale_log2;
  int bidir;
  int acc;            // add to the dk and dv that the residue pass wrote (the split backward)
};

// RES as for the dq pass: RES = 1 takes the skips alone in the residue-class view (the CTA's keys
// are keys u*pi + res of the sequence, read by the rows u + m0 .. u + S of the same class, all with
// the skip prior) and writes dk, dv; the window pass (S = 0) then adds to them.
template <int D, int RES>
__global__ void __launch_bounds__(KSmem<D>::kThreads, KSmem<D>::kCtas) bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmk,
                                                                        const __grid_constant__ CUtensorMap tmv,
                                                                        const __grid_constant__ CUtensorMap tmq,
                                                                        const __grid_constant__ CUtensorMap tmg,
                                                                        KParams prm) {
  using namespace tc;
  using L = KSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const sbase = smem_raw + (base - raw);
  if (base - raw + L::kTotal > (uint32_t)L::kAlloc) {
    if (threadIdx.x == 0) raise_error(kErrInternal);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int res = RES ? (int)(blockIdx.x % prm.pi) : 0;
  // this CTA's keys j0 .. j0 + 127 of the view (the sequence, or residue class res)
  const long long j0 = RES ? (long long)(blockIdx.x / prm.pi) * BM : (long long)blockIdx.x * BM;
  const long long T = RES ? prm.n / prm.pi : prm.n;  // rows of the view
  const uint32_t sK = base + L::kK, sV = base + L::kV, sQ = base + L::kQ, sG = base + L::kG;
  const uint32_t bar0 = base + L::kBar;
  const uint32_t bar_kv = bar0;
  auto bar_qfull = [&](int s) { return bar0 + 8u * (1 + s); };
  auto bar_qempty = [&](int s) { return bar0 + 8u * (1 + NSTAGE + s); };
  auto bar_gfull = [&](int s) { return bar0 + 8u * (1 + 2 * NSTAGE + s); };
  auto bar_gempty = [&](int s) { return bar0 + 8u * (1 + 3 * NSTAGE + s); };
  constexpr int NBUF = L::kNbuf;
  auto bar_sfull = [&](int b) { return bar0 + 8u * (1 + 4 * NSTAGE + b); };
  auto bar_pfull = [&](int b) { return bar0 + 8u * (1 + 4 * NSTAGE + NBUF + b); };
  auto bar_kvdone = [&](int b) { return bar0 + 8u * (1 + 4 * NSTAGE + 2 * NBUF + b); };
  const uint32_t bar_drain = bar0 + 8u * (1 + 4 * NSTAGE + 3 * NBUF);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(sbase + L::kMisc);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(sbase + L::kMisc + 4);

  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmk) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmv) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmq) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmg) : "memory");
    mbar_init(bar_kv, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_expect_tx(bar_kv, 2 * L::kKeyBytes);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      if (RES) {
        tma_load_4d(sK + c * BM * 128, &tmk, bar_kv, c * 64, res, (int)j0, bh);
        tma_load_4d(sV + c * BM * 128, &tmv, bar_kv, c * 64, res, (int)j0, bh);
      } else {
        tma_load_3d(sK + c * BM * 128, &tmk, bar_kv, c * 64, (int)j0, bh);
        tma_load_3d(sV + c * BM * 128, &tmv, bar_kv, c * 64, (int)j0, bh);
      }
    }
  }
  const int m0 = first_skip_m(prm.kwin, prm.pi);
  ReaderWalk walk;
  if (RES) {  // readers of view key u: rows u + m0 .. u + S
    walk.init_residue(j0, T, BM, prm.S, m0);
  } else {
    walk.init(j0, prm.n, BM, prm.kwin, prm.pi, prm.S, prm.bidir != 0);
  }
  int t_first = -1;
  auto load_rows = [&](uint32_t dst, const CUtensorMap* map, uint32_t bar, long long r0) {
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      if (RES)
        tma_load_4d(dst + c * BN * 128, map, bar, c * 64, res, (int)r0, bh);
      else
        tma_load_3d(dst + c * BN * 128, map, bar, c * 64, (int)r0, bh);
    }
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(bar_qfull(s), 1);
      mbar_init(bar_qempty(s), 1);
      mbar_init(bar_gfull(s), 1);
      mbar_init(bar_gempty(s), 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(bar_sfull(b), 1);
      mbar_init(bar_pfull(b), BM);
      mbar_init(bar_kvdone(b), 1);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    t_first = walk.next(0);
    if (t_first >= 0) {
      mbar_expect_tx(bar_qfull(0), L::kRowBytes);
      load_rows(sQ, &tmq, bar_qfull(0), (long long)t_first * BN);
      mbar_expect_tx(bar_gfull(0), L::kRowBytes);
      load_rows(sG, &tmg, bar_gfull(0), (long long)t_first * BN);
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "n"(L::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // pair b: S^T at b * 128, dP^T at b * 128 + 64; dV, dK after the pairs
  const uint32_t tdV = tmem + 2 * BN * NBUF, tdK = tdV + D;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      constexpr uint32_t kRow = L::kRowBytes;
      int nq = t_first >= 0 ? 1 : 0, ng = nq;
      for (int t = t_first >= 0 ? walk.next(t_first + 1) : -1; t >= 0; t = walk.next(t + 1)) {
        const int s = nq % NSTAGE, use = nq / NSTAGE;
        if (use > 0 && !mbar_wait(bar_qempty(s), (use - 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_qfull(s), kRow);
        load_rows(sQ + s * kRow, &tmq, bar_qfull(s), (long long)t * BN);
        ++nq;
        if (use > 0 && !mbar_wait(bar_gempty(s), (use - 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_gfull(s), kRow);
        load_rows(sG + s * kRow, &tmg, bar_gfull(s), (long long)t * BN);
        ++ng;
      }
      if (*abort_flag) {
        volatile int never = 0;
        mbar_wait(bar_kv, 0, &never);
        for (int u = nq > NSTAGE ? nq - NSTAGE : 0; u < nq; ++u)
          mbar_wait(bar_qfull(u % NSTAGE), (u / NSTAGE) & 1, &never);
        for (int u = ng > NSTAGE ? ng - NSTAGE : 0; u < ng; ++u)
          mbar_wait(bar_gfull(u % NSTAGE), (u / NSTAGE) & 1, &never);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kRow = L::kRowBytes;
      constexpr uint32_t idesc_s = idesc_bf16(BM, BN, 0);  // S^T, dP^T: B (Q, dO) K-major
      constexpr uint32_t idesc_a = idesc_bf16(BM, D, 1);   // dV, dK: B (dO, Q) N-major
      bool okw = mbar_wait(bar_kv, 0, abort_flag);
      tc_fence_after();
      // S^T = K Q^T, dP^T = V dO^T of row tile j into pair j % NBUF
      auto issue_s = [&](int j) -> bool {
        const int s = j % NSTAGE, b = j % NBUF;
        if (!mbar_wait(bar_qfull(s), (j / NSTAGE) & 1, abort_flag)) return false;
        if (!mbar_wait(bar_gfull(s), (j / NSTAGE) & 1, abort_flag)) return false;
        // the dV, dK MMAs of tile j - NBUF read P^T, dS^T over the columns overwritten here
        if (j >= NBUF && !mbar_wait(bar_kvdone(b), ((j - NBUF) / NBUF) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t tS = tmem + b * 2 * BN, tP = tS + BN;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t in = (kk & 3) * 32;
          tc_mma(tS, sw128_desc(sK + (kk >> 2) * (BM * 128) + in, 16, 1024),
                 sw128_desc(sQ + s * kRow + (kk >> 2) * (BN * 128) + in, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t in = (kk & 3) * 32;
          tc_mma(tP, sw128_desc(sV + (kk >> 2) * (BM * 128) + in, 16, 1024),
                 sw128_desc(sG + s * kRow + (kk >> 2) * (BN * 128) + in, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar_sfull(b));
        return true;
      };
      // dV += P^T dO and dK += dS^T Q of tile j: K = BN rows, 16 per instruction
      auto issue_kv = [&](int j) -> bool {
        const int s = j % NSTAGE, b = j % NBUF;
        if (!mbar_wait(bar_pfull(b), (j / NBUF) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t tS = tmem + b * 2 * BN, tP = tS + BN;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t acol = 16 * (kk >> 1) + 8 * (kk & 1);
          const uint32_t acc = (j == 0 && kk == 0) ? 0u : 1u;
          tc_mma_ts(tdV, tS + acol, sw128_desc(sG + s * kRow + kk * 16 * 128, BN * 128, 1024), idesc_a, acc);
          tc_mma_ts(tdK, tP + acol, sw128_desc(sQ + s * kRow + kk * 16 * 128, BN * 128, 1024), idesc_a, acc);
        }
        tc_commit(bar_kvdone(b));
        tc_commit(bar_qempty(s));
        tc_commit(bar_gempty(s));
        return true;
      };
      // one pair: dV, dK of tile j - 1, then S^T of tile j; two pairs: S^T of tile j first
      int jt = 0;
      for (int t = walk.next(0); okw; t = walk.next(t + 1), ++jt) {
        const bool have = t >= 0;
        if (NBUF == 1 && jt > 0 && !issue_kv(jt - 1)) break;
        if (have && !issue_s(jt)) break;
        if (NBUF == 2 && jt > 0 && !issue_kv(jt - 1)) break;
        if (!have) break;
      }
      tc_commit(bar_drain);
      volatile int never = 0;
      mbar_wait(bar_drain, 0, &never);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ key warpgroups
    const int wg = (warp - 2) >> 2;  // takes the row tiles j with j % NBUF == wg, in pair wg
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const long long j = j0 + r;  // key of the view
    const bool key_ok = j < T;
    const long long krow = (long long)bh * prm.n + (key_ok ? (RES ? j * prm.pi + res : j) : 0);
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    // rows reading j as window key (RES: the band of view rows j + m0 .. j + S, all skip readers)
    const long long w_lo = RES ? j + m0 : (prm.bidir ? (j - prm.kwin > 0 ? j - prm.kwin : 0) : j);
    const long long w_hi = RES ? (j + prm.S < T - 1 ? j + prm.S : T - 1)
                               : (j + prm.kwin < prm.n - 1 ? j + prm.kwin : prm.n - 1);
    KeyReaders kr;
    kr.init(j, prm.pi, RES ? 0 : prm.S, m0, walk.rpi, prm.bidir != 0, prm.n);
    const float NEG_INF = -INFINITY;
    const int tid = (threadIdx.x - 64) & 127;  // within the warpgroup
    float4* const stat = reinterpret_cast<float4*>(sbase + L::kStat) + wg * 2 * BN;
    const long long rbase = (long long)bh * prm.n;
    const uint32_t tS = tmem + wg * 2 * BN, tP = tS + BN;
    // (lse2, D, the band's prior, the skip prior) of row tid of the tile at r0: RES's band is skip
    // keys
    auto row_terms = [&](long long r0) -> float4 {
      const long long i = r0 + tid;  // row of the view
      const long long ri = rbase + (RES ? i * prm.pi + res : i);
      return i < T ? make_float4(prm.lse2[ri], prm.Dr[ri], RES ? prm.bp2[ri] : prm.bl2[ri], prm.bp2[ri])
                   : make_float4(0.f, 0.f, NEG_INF, NEG_INF);
    };
    // the group's next tile after t (the walk's next, or the one after it with two groups)
    auto next_own = [&](int t) -> int {
      int u = walk.next(t + 1);
      if (NBUF == 2 && u >= 0) u = walk.next(u + 1);
      return u;
    };
    bool ok = true;
    int jt = 0;
    float4 pre = make_float4(0.f, 0.f, NEG_INF, NEG_INF);  // the row terms of the group's next tile
    bool have_pre = false;
    for (int t = walk.next(0); t >= 0; t = walk.next(t + 1), ++jt) {
      if (jt % NBUF != wg) continue;
      const long long r0 = (long long)t * BN;
      // the tile's row terms into this tile's buffer of the warpgroup (the other buffer may still
      // be read by a warp on the group's previous tile; a warp here has finished that one); the
      // next tile's are loaded now, to land while this tile is processed
      float4* const st = stat + ((jt / NBUF) & 1) * BN;
      if (tid < BN) {
        st[tid] = have_pre ? pre : row_terms(r0);
        const int tn = next_own(t);
        if (tn >= 0) pre = row_terms((long long)tn * BN);
        have_pre = true;
      }
      asm volatile("bar.sync %0, 128;" ::"r"(1 + wg) : "memory");
      if (!ok) continue;  // keep taking part in the barrier above while the other warps finish
      if (!__all_sync(0xffffffffu, mbar_wait(bar_sfull(wg), (jt / NBUF) & 1, abort_flag))) {
        ok = false;
        continue;
      }
      tc_fence_after();
      const long long lo64 = w_lo - r0, hi64 = w_hi - r0;
      const int lc_lo = lo64 < 0 ? 0 : (lo64 > BN ? BN : (int)lo64);
      const int lc_hi = hi64 > BN - 1 ? BN - 1 : (hi64 < -1 ? -1 : (int)hi64);
      const uint64_t skw = kr.take(r0);
      // 16 rows at a time (registers): P^T and dS^T of rows c0 .. c0 + 15 go to the 8 packed
      // columns c0 / 2 .., which this loop has already read
      const uint64_t wm64 = key_ok ? (uint64_t)window_bits(lc_lo, lc_hi) | ((uint64_t)window_bits(lc_lo - 32, lc_hi - 32) << 32)
                                   : 0ull;
      const uint64_t sk64 = key_ok ? skw : 0ull;
#pragma unroll 1
      for (int cb = 0; cb < BN / 16; ++cb) {
        const int c0 = cb * 16;
        float x[16], g[16];
        tmem_ld16(tS + lane_off + c0, x);
        tmem_ld16(tP + lane_off + c0, g);
        const uint32_t wm = (uint32_t)(wm64 >> c0) & 0xFFFFu;
        const uint32_t skb = (uint32_t)(sk64 >> c0) & 0xFFFFu;
        uint32_t pk[8], dk2[8];
        if (__all_sync(0xffffffffu, (wm | skb) == 0u)) {
#pragma unroll
          for (int w = 0; w < 8; ++w) pk[w] = dk2[w] = 0u;
        } else {
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const float4 ra = st[c0 + e], rb = st[c0 + e + 1];
            const float b0 = ((wm >> e) & 1u) ? ra.z : (((skb >> e) & 1u) ? ra.w : NEG_INF);
            const float b1 = ((wm >> (e + 1)) & 1u) ? rb.z : (((skb >> (e + 1)) & 1u) ? rb.w : NEG_INF);
            const float p0 = ex2(fmaf(x[e], prm.scale_log2, b0 - ra.x));
            const float p1 = ex2(fmaf(x[e + 1], prm.scale_log2, b1 - rb.x));
            const float d0 = p0 * (g[e] - ra.y), d1 = p1 * (g[e + 1] - rb.y);
            __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1), db = __floats2bfloat162_rn(d0, d1);
            pk[e >> 1] = *reinterpret_cast<uint32_t*>(&pb);
            dk2[e >> 1] = *reinterpret_cast<uint32_t*>(&db);
          }
        }
        __syncwarp();
        tmem_st8(tS + lane_off + 8 * cb, pk);   // P^T over S^T columns already read
        tmem_st8(tP + lane_off + 8 * cb, dk2);  // dS^T over dP^T columns already read
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_pfull(wg));
    }
    // ---- epilogue: dk = tau dK, dv = dV (two warpgroups: dk from group 0, dv from group 1)
    // every MMA done: the drain barrier, committed once after the MMA warp's last issue (a pair's
    // own barrier could alias: a group that took none of the pair's last tiles cannot tell its
    // phases apart by parity)
    const bool have = __all_sync(0xffffffffu, ok && jt > 0 && mbar_wait(bar_drain, 0, abort_flag));
    if (have) tc_fence_after();
    const float tau = prm.scale_log2 / kLog2e;
    auto write_rows = [&](uint32_t tacc, float* dst, float scale) {
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float4* p = reinterpret_cast<float4*>(dst + krow * D + c * 32);
        float4 prev[8];  // the residue pass's dk or dv, loaded before the TMEM read to overlap it
        if (!RES && prm.acc && key_ok) {
#pragma unroll
          for (int e = 0; e < 8; ++e) prev[e] = p[e];
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) prev[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float a[32];
        if (have) {
          tmem_ld32(tacc + lane_off + c * 32, a);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) a[e] = 0.f;
        }
        if (key_ok) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 u = prev[e];
            p[e] = make_float4(u.x + scale * a[4 * e], u.y + scale * a[4 * e + 1], u.z + scale * a[4 * e + 2],
                               u.w + scale * a[4 * e + 3]);
          }
        }
      }
    };
    if (have || jt == 0) {
      if (NBUF == 1 || wg == 0) write_rows(tdK, prm.dk, tau);
      if (NBUF == 1 || wg == 1) write_rows(tdV, prm.dv, 1.f);
    }
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(L::kTmemCols) : "memory");
  }
}

// The row-side tensor maps: the sequence view, or (RES) the residue-class view, box_rows rows a box.
template <int RES>
inline bool bwd_map(CUtensorMap* m, const void* p, int BH, int n, int d, int pi, int box_rows) {
  return RES ? tc::make_residue_map(m, p, BH, n, d, pi, box_rows) : tc::make_map(m, p, BH, n, d, box_rows);
}

// Grid columns: the 128-row (or key) tiles of the view; RES: pi classes of n / pi rows each.
template <int RES>
inline unsigned bwd_tiles(int n, int pi) {
  return RES ? (unsigned)(pi * ((n / pi + BM - 1) / BM)) : (unsigned)((n + BM - 1) / BM);
}

template <int D, int RES>
cudaError_t launch_bwd_dkv(const void* q, const void* k, const void* v, const void* dout, const KParams& p, int BH,
                           cudaStream_t st, const char** why) {
  CUtensorMap mk, mv, mq, mg;
  if (!bwd_map<RES>(&mk, k, BH, p.n, D, p.pi, BM) || !bwd_map<RES>(&mv, v, BH, p.n, D, p.pi, BM) ||
      !bwd_map<RES>(&mq, q, BH, p.n, D, p.pi, BN) || !bwd_map<RES>(&mg, dout, BH, p.n, D, p.pi, BN)) {
    *why = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(bwd_dkv_kernel<D, RES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         KSmem<D>::kAlloc);
    if (e != cudaSuccess) {
      *why = "cudaFuncSetAttribute";
      return e;
    }
    attr_done = true;
  }
  const dim3 grid(bwd_tiles<RES>(p.n, p.pi), (unsigned)BH);
  bwd_dkv_kernel<D, RES><<<grid, KSmem<D>::kThreads, KSmem<D>::kAlloc, st>>>(mk, mv, mq, mg, p);
  *why = "tensor-core dk/dv kernel launch";
  return cudaGetLastError();
}

template <int D, int RES>
cudaError_t set_bwd_smem_attr() {
  static bool done = false;
  if (done) return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(bwd_dq_kernel<D, RES>, cudaFuncAttributeMaxDynamicSharedMemorySize, BSmem<D>::kAlloc);
  if (e == cudaSuccess) done = true;
  return e;
}

// The dq pass: q, dout [BH, n, D] bf16, k, v [BH, n, D] bf16; lse, Dr [BH, n] from the forward.
template <int D, int RES>
cudaError_t launch_bwd_dq(const void* q, const void* k, const void* v, const void* dout, const BParams& p, int BH,
                          cudaStream_t st, const char** why) {
  CUtensorMap mq, mg, mk, mv;
  if (!bwd_map<RES>(&mq, q, BH, p.n, D, p.pi, BM) || !bwd_map<RES>(&mg, dout, BH, p.n, D, p.pi, BM) ||
      !bwd_map<RES>(&mk, k, BH, p.n, D, p.pi, BN) || !bwd_map<RES>(&mv, v, BH, p.n, D, p.pi, BN)) {
    *why = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  cudaError_t e = set_bwd_smem_attr<D, RES>();
  if (e != cudaSuccess) {
    *why = "cudaFuncSetAttribute";
    return e;
  }
  const dim3 grid(bwd_tiles<RES>(p.n, p.pi), (unsigned)BH);
  bwd_dq_kernel<D, RES><<<grid, BSmem<D>::kThreads, BSmem<D>::kAlloc, st>>>(mq, mg, mk, mv, p);
  *why = "tensor-core dq kernel launch";
  return cudaGetLastError();
}

}  // namespace tcb
}  // namespace pia
