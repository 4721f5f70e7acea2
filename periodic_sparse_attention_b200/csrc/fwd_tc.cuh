// fwd_tc.cuh -- pi-attention prefill on Blackwell tensor cores (tcgen05 + TMEM + TMA), bf16,
// head size 64 or 128.
//
// Work unit: one CTA per (query tile of 128 rows, b, h).  The keys a tile needs are the union of
// its window band [i0 - k, i0 + 127] and, for every surviving skip m, the block
// [i0 - m*pi, i0 + 127 - m*pi]; the CTA walks the 64-key tiles that intersect this union in
// increasing order ("local sweep" and "periodic gather" of the method's execution schedule, both
// as tile loads) and evaluates every tile with the tensor cores:
//
//   TMA producer warp   Q tile once, then K and V tiles into a ring (four stages at d = 64, two at
//                       d = 128; 128B swizzle)
//   MMA warp            S = Q K^T (128 x 64, fp32 in TMEM), then O += P V (128 x d, fp32 in TMEM)
//   softmax warpgroup   one thread per query row: reads its S row from TMEM, applies the index
//                       rule as a mask and the gate as a log-prior (log(alpha) on window keys,
//                       log(1 - alpha) on skip keys, -inf elsewhere), keeps one running max and
//                       one running sum for the whole union (a single softmax), writes P (bf16)
//                       back into TMEM over the S columns it has read, where the P.V MMA takes
//                       its A operand; at the end divides O by the sum and writes out and lse.
//
// Online softmax with a lazy reference: probabilities are taken against a reference max that is
// only raised when a tile's max exceeds it by more than 2^8, so O (in TMEM) is rescaled rarely;
// every probability stays <= 2^8 and the final division uses the same reference, so the result
// is exact up to rounding.
//
// Every wait on an mbarrier is bounded (pia::kWaitLimitCycles).  A wait that gives up sets the device
// error word and an abort flag in shared memory; all roles then leave their loops, drain their
// own asynchronous work (bounded again) and the CTA frees its TMEM and exits.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tile_rule.cuh"

namespace pia {
namespace tc {

constexpr int BM = 128;        // query rows per CTA
constexpr int BN = kTileKeys;  // keys per tile (64)
// Pipeline shape.  Both head sizes run two CTAs per SM and one softmax warpgroup per CTA; TMEM per
// CTA is 256 columns: S buffers of 64 columns (the next tile's Q.K^T runs while the softmax works
// on this one; P is written back over the S columns it has read) -- three for D = 64, two for
// D = 128 -- and O (D columns).  Shared memory: the Q tile (128 rows) and a ring of 64-row K and
// V tiles, four stages at D = 64 (the loads of the tiles after next are in flight while this one
// is worked on) and two at D = 128 (where two CTAs an SM leave room for no more).  The K stages,
// and the V stages, are each one contiguous region of at least 128 rows, which the epilogue
// reuses.
// (Two warpgroups splitting each S row by columns also fit, at 96 registers a thread, but the
// per-tile exchange of their row maxima cost more than the halved pass over the row saved.)
template <int D> constexpr int kNstage = D == 64 ? 4 : 2;  // K/V ring depth
// S buffers in TMEM: the Q.K^T of tile j needs the P.V of tile j - NSB finished (P sits in the
// buffer it overwrites), so a third buffer gives that P.V a whole softmax pass of slack; it fits
// the 256 columns of a CTA only next to a 64-column O.
template <int D> constexpr int kNsb = D == 64 ? 3 : 2;
template <int D> constexpr int kCtasPerSm = 2;
constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 softmax (one query row a thread)
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// ---- shared memory plan (offsets from a 1024-byte aligned base) ---------------------------------
template <int D>
struct Smem {
  static constexpr int NSTAGE = kNstage<D>;
  static constexpr int kQBytes = BM * D * 2;             // the Q tile (bf16)
  static constexpr int kKVBytes = BN * D * 2;            // one K or V tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;
  static constexpr int kV = kK + NSTAGE * kKVBytes;
  static constexpr int kBar = kV + NSTAGE * kKVBytes;    // (P lives in TMEM, over its S columns)
  static constexpr int kTmemCols = 256;                  // S buffers (BN each) + O (D)
  static constexpr int NSB = kNsb<D>;
  static_assert(NSB * BN + D <= kTmemCols && kTmemCols * kCtasPerSm<D> <= 512, "TMEM columns");
  static_assert(NSTAGE * kKVBytes >= kQBytes, "the K and V regions each hold one 128-row tile");
  // barriers: q_full, k_full[NSTAGE], k_empty[NSTAGE], v_full[NSTAGE], v_empty[NSTAGE],
  // s_full[NSB], pv_done[NSB], p_full[NSB], drain, skip partials
  static constexpr int kNumBars = 1 + 4 * NSTAGE + 3 * NSB + 2;
  static constexpr int kMisc = kBar + kNumBars * 8;      // tmem base (4 B), abort flag (4 B)
  static constexpr int kWg = (kMisc + 8 + 15) / 16 * 16; // w_g[h] staging, D floats (read as float4)
  static constexpr int kTotal = kWg + D * 4;
  static_assert(kQ % 1024 == 0 && kK % 1024 == 0 && kV % 1024 == 0 && kKVBytes % 1024 == 0,
                "128-byte-swizzled tiles sit on 1 KB");
  static_assert(kBar % 8 == 0 && kWg % 16 == 0, "mbarriers on 8 bytes, the w_g staging on 16");
  static constexpr int kAlloc = kTotal + 1024 - 128;     // slack to align a (>= 128 B aligned) base to 1 KB
  // 228 KB of shared memory per SM, 1 KB of it reserved per CTA
  static_assert(kAlloc <= 228 * 1024 / kCtasPerSm<D> - 1024, "shared memory of the CTAs on one SM");
};

// ---- PTX wrappers ------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// One bounded wait step: try_wait without a suspend-time hint, so the thread waits for a short,
// system-defined time before returning false (a hint of milliseconds measurably delayed wake-ups).
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false when the limit passed or another thread of the CTA aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      raise_error(kErrWaitTimeout);
      *abort_flag = 1;
      return false;
    }
  }
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, "
      "%6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}
__device__ __forceinline__ void tma_store_commit_and_wait_read() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The same with A (M x K, bf16 packed two per 32-bit column, one row per lane) read from TMEM.
__device__ __forceinline__ void tc_mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// 32 consecutive TMEM columns of this warp's 32 lanes: lane l gets row (32*(warp%4) + l).  The
// wait is inside the same asm statement so no use of the results can be scheduled before it.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(r[t]);
}
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* v) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int t = 0; t < 64; ++t) v[t] = __uint_as_float(r[t]);
}
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, float* v) {
  uint32_t r[128];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, %96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int t = 0; t < 128; ++t) v[t] = __uint_as_float(r[t]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int t = 0; t < 16; ++t) v[t] = __uint_as_float(r[t]);
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// log(sigmoid(x)) = min(x, 0) - log(1 + e^-|x|) from the fast exponential and logarithm: the
// absolute error (~1e-7) is far below what the priors need, and the precise library versions are
// on the critical path of every CTA.
__device__ __forceinline__ float log_sigmoid_fast(float x) {
  return fminf(x, 0.f) - __logf(1.f + __expf(-fabsf(x)));
}


// v[k] for a run-time k in 0..31 from a register array: a 5-level tree of selects on the bits of
// k (independent selects, no local memory, no long dependency chain).
__device__ __forceinline__ float pick32(const float* v, int k) {
  float a[16], b[8], c[4], d[2];
  const bool k0 = k & 1, k1 = k & 2, k2 = k & 4, k3 = k & 8, k4 = k & 16;
#pragma unroll
  for (int e = 0; e < 16; ++e) a[e] = k0 ? v[2 * e + 1] : v[2 * e];
#pragma unroll
  for (int e = 0; e < 8; ++e) b[e] = k1 ? a[2 * e + 1] : a[2 * e];
#pragma unroll
  for (int e = 0; e < 4; ++e) c[e] = k2 ? b[2 * e + 1] : b[2 * e];
#pragma unroll
  for (int e = 0; e < 2; ++e) d[e] = k3 ? c[2 * e + 1] : c[2 * e];
  return k4 ? d[1] : d[0];
}


// max of three (one instruction on sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ---- UMMA descriptors ----------------------------------------------------------------------------
// Shared-memory matrix descriptor (sm_100): start address >> 4 in bits [0,14), leading byte
// offset >> 4 in [16,30), stride byte offset >> 4 in [32,46), version 1 in [46,48), layout type
// in [61,64) (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) | ((uint64_t)(sbo >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, A K-major, B K-major
// (b_mn_major = 0) or N-major (1), N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Three ways to run the kernel:
//   kFused      window and skips of a 128-row query tile in one pass (the default)
//   kResidue    the skip part alone, in the residue-class view: for a residue r (mod pi), rows
//               t*pi + r form their own sequence, and P(i) becomes the band t - S .. t - m0 of it,
//               a dense band the tensor cores evaluate without the 1/128 diagonal waste of skip
//               tiles.  Writes the skip partial (normalised output in bf16, lse in fp32) of every
//               row to scratch, in sequence layout.
//   kBandMerge  the window part alone; the epilogue merges the skip partial of its rows:
//               with a = log2 of the window mass, b = log2 of the skip mass, M = max(a, b),
//               out = (out_L 2^(a-M) + out_P 2^(b-M)) / (2^(a-M) + 2^(b-M)),
//               lse = (M + log2(2^(a-M) + 2^(b-M))) ln 2 -- the same single softmax, summed in
//               two pieces.
enum : int { kFused = 0, kResidue = 1, kBandMerge = 2 };

struct Params {
  const float* w_g;
  const float* b_g;
  __nv_bfloat16* out;
  float* lse;
  __nv_bfloat16* skip_o;  // [B*H, n, D] skip partial (kResidue writes, kBandMerge reads)
  float* skip_lse;        // [B*H, n]
  int H, n, kwin, pi, S;
  int T;                  // kResidue: rows per residue class (n / pi)
  float scale_log2;
  int bidir;              // the bidirectional index rule (two-sided window, forward skips; kResidue: both bands)
  int tile0;              // kFused, kBandMerge: query tile of the grid's first CTA
  // kFused over one shard of a longer sequence: q/out/lse row r is sequence row row0 + r; k/v
  // row r is sequence row kv0 + r (the index rule runs in sequence rows).  0 and 0 otherwise.
  long long row0, kv0;
  // For the backward (kFused, kBandMerge): with dout given, the epilogue also writes
  // Dout[row] = dout . out from the fp32 output row (before its rounding to bf16).  Null otherwise.
  const __nv_bfloat16* dout;
  float* Dout;
  // For the backward too (kFused, kBandMerge; null otherwise): the row terms its dk/dv pass reads,
  // lse in log2 units (from the stored natural-log value) and the log2 priors log2(alpha) and
  // log2(1 - alpha).
  float* lse2;
  float* bl2;
  float* bp2;
};

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, kCtasPerSm<D>) fwd_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                                                                          const __grid_constant__ CUtensorMap tmk,
                                                                          const __grid_constant__ CUtensorMap tmv,
                                                                          const __grid_constant__ CUtensorMap tmo,
                                                                          const __grid_constant__ CUtensorMap tms,
                                                                          Params prm) {
  using L = Smem<D>;
  constexpr int NSB = kNsb<D>;
  constexpr int NSTAGE = L::NSTAGE;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const sbase = smem_raw + (base - raw);
  if (base - raw + L::kTotal > (uint32_t)L::kAlloc) {  // the plan does not fit: refuse, touch nothing
    if (threadIdx.x == 0) raise_error(kErrInternal);
    return;
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int h = bh % prm.H;
  // Thread 0 starts the Q tile's load before anything else: its latency (HBM, plus the tensor
  // map's first use) heads every CTA's critical path.  The tensor maps are prefetched meanwhile.
  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmq) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmk) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmv) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmo) : "memory");
    if (MODE == kBandMerge) asm volatile("prefetch.tensormap [%0];" ::"l"(&tms) : "memory");
    const uint32_t bq = base + L::kBar;  // bar_q
    mbar_init(bq, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_expect_tx(bq, L::kQBytes);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      if (MODE == kResidue)
        tma_load_4d(base + L::kQ + c * BM * 128, &tmq, bq, c * 64, (int)(blockIdx.x % prm.pi),
                    (int)(blockIdx.x / prm.pi) * BM, bh);
      else
        tma_load_3d(base + L::kQ + c * BM * 128, &tmq, bq, c * 64, (prm.tile0 + (int)blockIdx.x) * BM, bh);
    }
  }
  const int m0 = first_skip_m(prm.kwin, prm.pi);
  // query tile: rows q0 .. q0+127 of the view (the sequence, or residue class `res`)
  int res = 0;
  long long q0;
  TileWalk walk;
  if (MODE == kResidue) {
    res = blockIdx.x % prm.pi;
    q0 = (long long)(blockIdx.x / prm.pi) * BM;
    // keys of row t: t - S .. t - m0 (the skips of sequence row t*pi + res).  The walk runs in
    // periods of the whole sequence: a shard's rows start at period row0 / pi (whole periods)
    walk.init_residue(q0 + prm.row0 / prm.pi, prm.T + prm.row0 / prm.pi, BM, prm.S, m0, prm.bidir != 0);
  } else {
    q0 = (long long)(prm.tile0 + (int)blockIdx.x) * BM;
    walk.init(prm.row0 + q0, prm.row0 + prm.n, BM, prm.kwin, prm.pi, MODE == kFused ? prm.S : 0, prm.bidir != 0);
  }
  const int view_rows = MODE == kResidue ? prm.T : prm.n;
  // the k/v buffer's first row, in the walk's units (sequence rows; kResidue: periods)
  const long long kv_off = MODE == kResidue ? prm.kv0 / prm.pi : prm.kv0;
  // every thread walks the tiles with its own cursor (no division per step); thread 0 takes the
  // first tile at barrier init and goes on from there as the producer
  TileCursor cur;
  cur.init(walk);
  int t_first = -1;

  const uint32_t sQ = base + L::kQ, sK = base + L::kK, sV = base + L::kV;
  // P of tile j sits in TMEM over the columns of S buffer j % NSB that the softmax has read: the
  // 32-key chunk cb of P (16 packed columns) at column 16 cb of the buffer, written after S chunk
  // cb (columns 32 cb .. 32 cb + 31) has been read.
  const uint32_t bar0 = base + L::kBar;
  const uint32_t bar_q = bar0;
  auto bar_kfull = [&](int s) { return bar0 + 8u * (1 + s); };
  auto bar_kempty = [&](int s) { return bar0 + 8u * (1 + NSTAGE + s); };
  auto bar_vfull = [&](int s) { return bar0 + 8u * (1 + 2 * NSTAGE + s); };
  auto bar_vempty = [&](int s) { return bar0 + 8u * (1 + 3 * NSTAGE + s); };
  auto bar_sfull = [&](int b) { return bar0 + 8u * (1 + 4 * NSTAGE + b); };
  auto bar_pvdone = [&](int b) { return bar0 + 8u * (1 + 4 * NSTAGE + NSB + b); };  // P.V of buffer b
  // P of buffer b written by all 128 rows.  One barrier per buffer: with two buffers a fast warp
  // can finish the next tile before a slow one finishes this tile, and on a shared barrier its
  // arrivals would complete this tile's phase early.  No phase can run two ahead of a slow warp:
  // the tile after next in a buffer needs its Q.K^T, which waits for this tile's P.V, which waits
  // for every row's P.
  auto bar_pfull = [&](int b) { return bar0 + 8u * (1 + 4 * NSTAGE + 2 * NSB + b); };
  const uint32_t bar_drain = bar0 + 8u * (1 + 4 * NSTAGE + 3 * NSB);
  const uint32_t bar_so = bar_drain + 8;  // kBandMerge: the tile of skip partials has landed
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(sbase + L::kMisc);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(sbase + L::kMisc + 4);

  // one tile of `rows` rows of the view (r0 ..) into shared memory: D/64 boxes of 64 columns,
  // each rows x 128 bytes (the map's box has `rows` rows: BM for Q, BN for K and V)
  auto load_tile = [&](uint32_t dst, const CUtensorMap* map, uint32_t bar, long long r0, int rows) {
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      if (MODE == kResidue)
        tma_load_4d(dst + c * rows * 128, map, bar, c * 64, res, (int)r0, bh);
      else
        tma_load_3d(dst + c * rows * 128, map, bar, c * 64, (int)r0, bh);
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(bar_kfull(s), 1);
      mbar_init(bar_kempty(s), 1);
      mbar_init(bar_vfull(s), 1);
      mbar_init(bar_vempty(s), 1);
    }
    for (int b = 0; b < NSB; ++b) {
      mbar_init(bar_sfull(b), 1);
      mbar_init(bar_pvdone(b), 1);
      mbar_init(bar_pfull(b), BM);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_so, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    // the first K/V tile waits for nothing either: it starts now, before the TMEM allocation
    // and the block barrier
    t_first = cur.next();
    if (t_first >= 0) {
      mbar_expect_tx(bar_kfull(0), L::kKVBytes);
      load_tile(sK, &tmk, bar_kfull(0), (long long)t_first * BN - kv_off, BN);
      mbar_expect_tx(bar_vfull(0), L::kKVBytes);
      load_tile(sV, &tmv, bar_vfull(0), (long long)t_first * BN - kv_off, BN);
    }
  }
  if (warp == 1) {  // TMEM: S buffer b in columns [BN b, BN b + BN), O in [BN NSB, BN NSB + D)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "n"(L::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + BN * NSB;  // S buffer b at tS + BN b

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      constexpr uint32_t kKV = L::kKVBytes;
      int nk = t_first >= 0 ? 1 : 0, nv = nk;  // K and V tile loads issued (the first one at the start)
      for (int t = cur.next(); t >= 0; t = cur.next()) {
        const int s = nk % NSTAGE, use = nk / NSTAGE;
        if (use > 0 && !mbar_wait(bar_kempty(s), (use - 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_kfull(s), kKV);
        load_tile(sK + s * kKV, &tmk, bar_kfull(s), (long long)t * BN - kv_off, BN);
        ++nk;
        if (use > 0 && !mbar_wait(bar_vempty(s), (use - 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_vfull(s), kKV);
        load_tile(sV + s * kKV, &tmv, bar_vfull(s), (long long)t * BN - kv_off, BN);
        ++nv;
      }
      // kBandMerge: the 128-row tile of skip partials goes into the K region as soon as the last
      // Q.K^T has completed (its commit covers every earlier one), so that its load overlaps the
      // last tile's softmax and P.V
      bool so_issued = false;
      if (MODE == kBandMerge && !*abort_flag) {
        const int u = nk - 1;  // last K load
        if (u < 0 || mbar_wait(bar_kempty(u % NSTAGE), (u / NSTAGE) & 1, abort_flag)) {
          mbar_expect_tx(bar_so, L::kQBytes);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) tma_load_3d(sK + c * BM * 128, &tms, bar_so, c * 64, (int)q0, bh);
          so_issued = true;
        }
      }
      if (*abort_flag) {  // let the loads already in flight land before the CTA can exit
        volatile int never = 0;
        mbar_wait(bar_q, 0, &never);
        if (so_issued) mbar_wait(bar_so, 0, &never);
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
      constexpr uint32_t idesc_qk = idesc_bf16(BM, BN, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(BM, D, 1);
      bool okw = mbar_wait(bar_q, 0, abort_flag);
      tc_fence_after();
      // S_j = Q K_j^T into S buffer j % NSB : K = D, 16 per instruction; the operands' 64-column
      // blocks are BM x 128 B (Q) and BN x 128 B (K) apart
      auto issue_qk = [&](int s, int b) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t in = (kk & 3) * 32;
          tc_mma(tS + BN * b, sw128_desc(sQ + (kk >> 2) * (BM * 128) + in, 16, 1024),
                 sw128_desc(sK + s * kKV + (kk >> 2) * (BN * 128) + in, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // O += P V_j : K = BN keys, 16 per instruction; V is N-major (d contiguous, 64-column
      // blocks BN x 128 B apart)
      auto issue_pv = [&](int s, int b, bool first) {  // A = P from TMEM (S buffer b)
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t acol = BN * b + 16 * (kk >> 1) + 8 * (kk & 1);
          const uint32_t boff = kk * 16 * 128;
          tc_mma_ts(tO, tS + acol, sw128_desc(sV + s * kKV + boff, BN * 128, 1024), idesc_pv,
                    (first && kk == 0) ? 0u : 1u);
        }
      };
      // Q.K^T of tile j needs its K stage loaded and the P.V of tile j - NSB finished: that P.V
      // reads P from the columns this Q.K^T overwrites (MMAs into different accumulators are not
      // ordered with each other), and it was issued only once every row had written its P, so
      // the softmax is done with the buffer too.
      auto try_qk = [&](int jq) -> bool {
        const int s = jq % NSTAGE, b = jq % NSB;
        if (!mbar_wait(bar_kfull(s), (jq / NSTAGE) & 1, abort_flag)) return false;
        if (jq >= NSB && !mbar_wait(bar_pvdone(b), (jq / NSB - 1) & 1, abort_flag)) return false;
        tc_fence_after();
        issue_qk(s, b);
        tc_commit(bar_sfull(b));
        tc_commit(bar_kempty(s));
        return true;
      };
      int j = 0;
      int t = cur.next();
      if (okw && t >= 0) okw = try_qk(0);
      // The next tile's Q.K^T goes first: it runs while the softmax works on this tile.
      while (okw && t >= 0) {
        const int tn = cur.next();
        const int s = j % NSTAGE;
        if (tn >= 0 && !try_qk(j + 1)) break;
        if (!mbar_wait(bar_vfull(s), (j / NSTAGE) & 1, abort_flag)) break;
        if (!mbar_wait(bar_pfull(j % NSB), (j / NSB) & 1, abort_flag)) break;
        tc_fence_after();
        issue_pv(s, j % NSB, j == 0);
        tc_commit(bar_pvdone(j % NSB));
        tc_commit(bar_vempty(s));
        ++j;
        t = tn;
      }
      // all MMAs issued by this thread have completed once the drain barrier flips
      tc_commit(bar_drain);
      volatile int never = 0;
      mbar_wait(bar_drain, 0, &never);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax warpgroup
    constexpr int CPT = BN / 32;              // 32-column chunks of S (and of P) per tile
    const int q4 = warp & 3;                  // TMEM lane quarter this warp may access
    const int r = q4 * 32 + lane;             // query row within the tile
    const long long qi = q0 + r;              // row in the view
    const long long i = MODE == kResidue ? qi * prm.pi + res : prm.row0 + qi;  // row in the sequence (kResidue:
                                                                               // in the q buffer)
    const long long qg = MODE == kResidue ? qi + prm.row0 / prm.pi : qi;      // kResidue: period of the row
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    // kBandMerge: this row's skip-partial lse (written by the residue pass), loaded now so that
    // the epilogue does not wait for it
    const float skip_lse_row =
        MODE == kBandMerge && qi < view_rows ? prm.skip_lse[(long long)bh * prm.n + qi] : 0.f;

    // the row's keys, tile by tile: window columns from the window's bounds, skip columns from
    // the row's own skip keys taken in order (the residue pass: keys qi - S .. qi - m0 of its
    // view, no skips).  Set up while the Q tile is still in flight.
    const long long w_lo = MODE == kResidue ? (qg - prm.S > 0 ? qg - prm.S : 0) : (i - prm.kwin > 0 ? i - prm.kwin : 0);
    const long long w_hi = MODE == kResidue ? qg - m0
                           : prm.bidir ? (i + prm.kwin < prm.n - 1 ? i + prm.kwin : prm.n - 1)
                                       : i;
    // kResidue, bidirectional: the forward band qi + m0 .. qi + S of the view, carried as skip bits
    // (in this pass every key takes the skip prior, so the bits and the window columns weigh alike)
    const long long f_lo = qi + m0, f_hi = qi + prm.S < view_rows - 1 ? qi + prm.S : view_rows - 1;
    const bool fwd_band = MODE == kResidue && prm.bidir && prm.S >= m0;
    RowSkips rs;
    rs.init(i, prm.pi, MODE == kFused ? prm.S : 0, m0, walk.rpi, MODE == kFused && prm.bidir, prm.n);

    // gate on the unscaled query row.  w_g[h] is staged in shared memory while the Q tile is
    // still in flight.
    float* const wg_s = reinterpret_cast<float*>(sbase + L::kWg);
    if (threadIdx.x - 64 < D) wg_s[threadIdx.x - 64] = prm.w_g[(long long)h * D + (threadIdx.x - 64)];
    float z = prm.b_g[h];  // in flight with the w_g staging and the Q load
    asm volatile("bar.sync 1, 128;" ::: "memory");
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar_q, 0, abort_flag));
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

    // the prior of the keys this pass unmasks as "window" columns
    const float bias_l = log_sigmoid_fast(MODE == kResidue ? -z : z) * kLog2e;  // log2(alpha), or log2(1-alpha)
    const float bias_p = log_sigmoid_fast(-z) * kLog2e;                         // log2(1 - alpha)
    const float NEG_INF = -INFINITY;

    float m_ref = NEG_INF;  // reference max (log2 units)
    float l_sum = 0.f;      // running sum of probabilities against m_ref (fp32 values: for lse)
    float l_rnd = 0.f;      // the same sum of their bf16 roundings (the weights in P.V: for out)
    int j = 0;
    for (int t = cur.next(); ok && t >= 0; t = cur.next(), ++j) {
      const int sb = j % NSB;
      // every lane of the warp takes the same branch: tcgen05.ld is .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(bar_sfull(sb), (j / NSB) & 1, abort_flag))) { ok = false; break; }
      tc_fence_after();
      const uint32_t tSb = tS + BN * sb + lane_off;
      // the index rule on this tile, for row qi: window columns [lc_lo, lc_hi], skip columns bitmask
      const long long j0 = (long long)t * BN;
      const long long lo64 = w_lo - j0, hi64 = w_hi - j0;
      const int lc_lo = lo64 < 0 ? 0 : (lo64 > BN ? BN : (int)lo64);
      const int lc_hi = hi64 > BN - 1 ? BN - 1 : (hi64 < -1 ? -1 : (int)hi64);
      static_assert(BN == 64, "one 64-bit word of skip bits per tile");
      uint64_t skw = rs.take(j0);
      if (fwd_band) {  // columns of the forward band [f_lo, f_hi] in this tile
        const long long a = f_lo - j0, b = f_hi - j0;
        if (a <= BN - 1 && b >= 0 && a <= b) {
          const int lo = a < 0 ? 0 : (int)a, hi = b > BN - 1 ? BN - 1 : (int)b;
          skw = (hi == BN - 1 ? ~0ull : ((1ull << (hi + 1)) - 1ull)) & ~((1ull << lo) - 1ull);
        }
      }
      const uint32_t sk[2] = {(uint32_t)skw, (uint32_t)(skw >> 32)};
      const bool has_win = lc_lo <= lc_hi;
      uint32_t sk_any = 0u;
#pragma unroll
      for (int w = 0; w < BN / 32; ++w) sk_any |= sk[w];
      const bool has_skip = sk_any != 0u;

      // Pass 1: a reference for the tile, from the whole S row in one load: the max of the raw
      // scores, scaled, plus the larger prior present.  It bounds the true max of the biased
      // logits from above, and not by much: a key can only beat a key of higher prior by scoring
      // at least the prior gap more, so the bound exceeds the true max by at most twice the score
      // spread of the row.  Probabilities only need a reference at or above their max.
      float mt;
      float srow[BN];  // the S row as pass 1 loads it; pass 2 reuses it when the row is all window
      tmem_ld64(tSb, srow);
      {
        const float* x = srow;
        static_assert(BN == 64, "pass 1 reduces eight groups of eight columns");
        float mx[8];  // mx[e]: max over columns e, e + 8, ..., e + 56
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float m = max3f(x[e], x[8 + e], x[16 + e]);
          m = max3f(m, x[24 + e], x[32 + e]);
          m = max3f(m, x[40 + e], x[48 + e]);
          mx[e] = fmaxf(m, x[56 + e]);
        }
        const float mraw = max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
        const float top = has_win ? (has_skip ? fmaxf(bias_l, bias_p) : bias_l) : bias_p;
        mt = (has_win || has_skip) ? fmaf(mraw, prm.scale_log2, top) : NEG_INF;
      }

      // lazy reference max
      float factor = 1.f;
      bool rescale = false;
      if (mt > m_ref + kRescaleThreshold || (m_ref == NEG_INF && mt != NEG_INF)) {
        factor = ex2(m_ref - mt);  // 0 when m_ref = -inf
        rescale = m_ref != NEG_INF;  // O holds earlier tiles' sums
        l_sum *= factor;
        l_rnd *= factor;
        m_ref = mt;
      }
      const float m_use = m_ref == NEG_INF ? 0.f : m_ref;
      const float bl_m = bias_l - m_use, bp_m = bias_p - m_use;
      float ls = 0.f, lr = 0.f;

      if (__all_sync(0xffffffffu, lc_lo == 0 && lc_hi == BN - 1 && !has_skip)) {
        // Every row of the warp reads the whole tile as window keys (the inside of the band):
        // pass 2 from pass 1's registers, all 64 columns as one batch of independent work, and P
        // over S columns 0..31 in one store (the whole S row has been read).  Per pair of columns:
        // one packed FMA (scale and prior), two exponentials, one pack to bf16x2, and packed adds
        // into the fp32 sum and into the sum of the bf16 roundings.
        uint32_t pk[BN / 2];
        unsigned long long sp[4], sr[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) sp[a] = sr[a] = 0ull;
        const unsigned long long sc2 = f2pack(prm.scale_log2, prm.scale_log2), bb = f2pack(bl_m, bl_m);
#pragma unroll
        for (int e = 0; e < BN; e += 2) {
          float t0, t1;
          f2unpack(f2fma(f2pack(srow[e], srow[e + 1]), sc2, bb), t0, t1);
          const float p0 = ex2(t0), p1 = ex2(t1);
          __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
          const uint32_t u = *reinterpret_cast<uint32_t*>(&b2);
          pk[e >> 1] = u;
          sp[(e >> 1) & 3] = f2add(sp[(e >> 1) & 3], f2pack(p0, p1));
          sr[(e >> 1) & 3] = f2add(sr[(e >> 1) & 3], f2pack(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u)));
        }
        tmem_st32u(tSb, pk);
        float a0, a1, r0, r1;
        f2unpack(f2add(f2add(sp[0], sp[1]), f2add(sp[2], sp[3])), a0, a1);
        f2unpack(f2add(f2add(sr[0], sr[1]), f2add(sr[2], sr[3])), r0, r1);
        ls = a0 + a1;
        lr = r0 + r1;
      } else if (__all_sync(0xffffffffu, !has_skip) && __any_sync(0xffffffffu, has_win)) {
        // Every row of the warp reads only window keys here, a contiguous range of columns
        // (the band's edges and the causal diagonal), and some row reads at least one: the same
        // batch from registers, with the columns outside the row's range set to -inf before the
        // exponential (p = 0 exactly).  A warp with no key at all takes the rolled path's zeros.
        const uint64_t wb = lc_lo > lc_hi ? 0ull : ((~0ull >> (BN - 1 - lc_hi)) & (~0ull << lc_lo));
        const uint32_t wlo = (uint32_t)wb, whi = (uint32_t)(wb >> 32);
        uint32_t pk[BN / 2];
        unsigned long long sp[4], sr[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) sp[a] = sr[a] = 0ull;
        const unsigned long long sc2 = f2pack(prm.scale_log2, prm.scale_log2), bb = f2pack(bl_m, bl_m);
#pragma unroll
        for (int e = 0; e < BN; e += 2) {
          float t0, t1;
          f2unpack(f2fma(f2pack(srow[e], srow[e + 1]), sc2, bb), t0, t1);
          const uint32_t wv = e < 32 ? wlo : whi;
          if (!((wv >> (e & 31)) & 1u)) t0 = NEG_INF;
          if (!((wv >> ((e + 1) & 31)) & 1u)) t1 = NEG_INF;
          const float p0 = ex2(t0), p1 = ex2(t1);
          __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
          const uint32_t u = *reinterpret_cast<uint32_t*>(&b2);
          pk[e >> 1] = u;
          sp[(e >> 1) & 3] = f2add(sp[(e >> 1) & 3], f2pack(p0, p1));
          sr[(e >> 1) & 3] = f2add(sr[(e >> 1) & 3], f2pack(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u)));
        }
        tmem_st32u(tSb, pk);
        float a0, a1, r0, r1;
        f2unpack(f2add(f2add(sp[0], sp[1]), f2add(sp[2], sp[3])), a0, a1);
        f2unpack(f2add(f2add(sr[0], sr[1]), f2add(sr[2], sr[3])), r0, r1);
        ls = a0 + a1;
        lr = r0 + r1;
      } else {
      // Pass 2, one 32-column chunk at a time (a rolled loop, re-reading the chunk from TMEM):
      // probabilities against the reference, P (bf16, two per column) back into TMEM, and two
      // row sums -- of the fp32
      // probabilities (for lse) and of their bf16 roundings (the weights P.V actually applies; the
      // output is normalised by this one, so a row of one key reproduces that key's value).
      //   no key in the chunk -> zeros; window keys only -> one FMA per logit; one skip key and
      //   no window key -> one exponential; otherwise window bits and skip bits pick each prior.
#pragma unroll 1
      for (int cb = 0; cb < CPT; ++cb) {
        const int c0 = cb * 32;
        float x[32];
        tmem_ld32(tSb + c0, x);
        const uint32_t skb = cb == 0 ? sk[0] : sk[CPT - 1];
        const uint32_t wm = window_bits(lc_lo - c0, lc_hi - c0);
        uint32_t pk[16];
        if ((wm | skb) == 0u) {
#pragma unroll
          for (int w = 0; w < 16; ++w) pk[w] = 0u;
        } else if (wm == 0u && (skb & (skb - 1u)) == 0u) {
          const int sc = __ffs(skb) - 1;
          const float p1 = ex2(fmaf(pick32(x, sc), prm.scale_log2, bp_m));
          __nv_bfloat162 b2 = __floats2bfloat162_rn(p1, p1);
          const uint32_t both = *reinterpret_cast<uint32_t*>(&b2);
          ls += p1;
          lr += __uint_as_float(both << 16);
          const uint32_t word = (sc & 1) ? (both & 0xFFFF0000u) : (both & 0x0000FFFFu);
#pragma unroll
          for (int w = 0; w < 16; ++w) pk[w] = (sc >> 1) == w ? word : 0u;
        } else {
          // per pair of columns: one packed FMA (scale and prior), two exponentials, one pack to
          // bf16x2, and packed adds into the fp32 sum and into the sum of the bf16 roundings
          // (unpacked from the bf16x2 word by two integer ops)
          unsigned long long sp[4], sr[4];
#pragma unroll
          for (int a = 0; a < 4; ++a) sp[a] = sr[a] = 0ull;
          const unsigned long long sc2 = f2pack(prm.scale_log2, prm.scale_log2);
          if (wm == 0xFFFFFFFFu && skb == 0u) {  // window keys only
            const unsigned long long bb = f2pack(bl_m, bl_m);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float t0, t1;
              f2unpack(f2fma(f2pack(x[e], x[e + 1]), sc2, bb), t0, t1);
              const float p0 = ex2(t0), p1 = ex2(t1);
              __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
              const uint32_t u = *reinterpret_cast<uint32_t*>(&b2);
              pk[e >> 1] = u;
              sp[(e >> 1) & 3] = f2add(sp[(e >> 1) & 3], f2pack(p0, p1));
              sr[(e >> 1) & 3] = f2add(sr[(e >> 1) & 3], f2pack(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u)));
            }
          } else {  // window edge and / or skip keys: each column's prior from its bits
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float b0 = (wm >> e) & 1u ? bl_m : ((skb >> e) & 1u ? bp_m : NEG_INF);
              const float b1 = (wm >> (e + 1)) & 1u ? bl_m : ((skb >> (e + 1)) & 1u ? bp_m : NEG_INF);
              float t0, t1;
              f2unpack(f2fma(f2pack(x[e], x[e + 1]), sc2, f2pack(b0, b1)), t0, t1);
              const float p0 = ex2(t0), p1 = ex2(t1);
              __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
              const uint32_t u = *reinterpret_cast<uint32_t*>(&b2);
              pk[e >> 1] = u;
              sp[(e >> 1) & 3] = f2add(sp[(e >> 1) & 3], f2pack(p0, p1));
              sr[(e >> 1) & 3] = f2add(sr[(e >> 1) & 3], f2pack(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u)));
            }
          }
          const unsigned long long sps = f2add(f2add(sp[0], sp[1]), f2add(sp[2], sp[3]));
          const unsigned long long srs = f2add(f2add(sr[0], sr[1]), f2add(sr[2], sr[3]));
          float a0, a1, r0, r1;
          f2unpack(sps, a0, a1);
          f2unpack(srs, r0, r1);
          ls += a0 + a1;
          lr += r0 + r1;
        }
        __syncwarp();  // rows may have taken different branches; tcgen05.st is .sync.aligned
        tmem_st16(tSb + 16 * cb, pk);  // over S columns already read
      }
      }
      l_sum += ls;
      l_rnd += lr;

      // (P.V of tile j - NSB, which read this buffer's P, has completed: the MMA thread waited for
      // it before the Q.K^T of this tile.  That also keeps the pv_done waits below unambiguous.)
      // The rescale comes after pass 2 (which does not touch O) so that the wait for the previous
      // P.V has had that time to complete; it must precede this tile's p_full arrival.
      if (__any_sync(0xffffffffu, rescale)) {
        // O must hold every earlier tile's P.V before it is rescaled: wait for the P.V of tile j - 1
        if (j >= 1 &&
            !__all_sync(0xffffffffu, mbar_wait(bar_pvdone((j - 1) % NSB), ((j - 1) / NSB) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the rescale is per row, but TMEM access is per warp: the warp rescales when any of its
        // rows needs it, the others multiply by 1
        const float f = rescale ? factor : 1.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(tO + lane_off + c * 32, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= f;
          tmem_st32(tO + lane_off + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      // the P.V of this tile may start; once it has finished, the buffer may take the Q.K^T of
      // tile j + NSB
      mbar_arrive(bar_pfull(sb));
    }
    // ---- epilogue: the normalised row goes to shared memory (the V region, free once the last
    // P.V has completed) in the 128-byte-swizzled 128-row tile layout, then one TMA store writes
    // the tile (rows past the end of the view are clipped by the tensor map).  kBandMerge merges
    // the tile of skip partials, which the producer has loaded into the K region.
    const bool row_ok = qi < view_rows;
    const long long orow = (long long)bh * prm.n + (MODE == kResidue ? i : qi);  // row in [B*H, n] layouts
    const bool have_o = __all_sync(
        0xffffffffu, ok && j > 0 && mbar_wait(bar_pvdone((j - 1) % NSB), ((j - 1) / NSB) & 1, abort_flag));
    const bool no_keys = MODE == kResidue && __all_sync(0xffffffffu, ok && j == 0);  // tile with no skip at all
    float lse_log2 = 0.f;
    if (have_o || no_keys) {
      if (have_o) tc_fence_after();
      bool so_ok = true;
      if (MODE == kBandMerge) so_ok = __all_sync(0xffffffffu, mbar_wait(bar_so, 0, abort_flag));
      float inv = l_rnd > 0.f ? 1.f / l_rnd : 0.f;
      float wl = 1.f, wp = 0.f, lse2 = m_ref + log2f(l_sum);  // log2 of this pass's mass
      if (MODE == kBandMerge && row_ok) {
        const float b2 = skip_lse_row * kLog2e;
        const float M = fmaxf(lse2, b2);
        wl = ex2(lse2 - M);
        wp = ex2(b2 - M);
        const float den = wl + wp;
        wl /= den;
        wp /= den;
        lse2 = M + log2f(den);
      }
      float o[D];  // the O row, one load
      if (have_o) {
        if (D == 128) tmem_ld128(tO + lane_off, o);
        else tmem_ld64(tO + lane_off, o);
      } else {
#pragma unroll
        for (int e = 0; e < D; ++e) o[e] = 0.f;
      }
      const unsigned long long ow2 = f2pack(inv * wl, inv * wl), wp2 = f2pack(wp, wp);
#pragma unroll
      for (int cl = 0; cl < D / 8; ++cl) {  // 16-byte chunk c of the row
        const int c = cl;
        const int blk = c >> 3, cc = c & 7;
        const uint32_t off = blk * (BM * 128) + r * 128 + ((cc ^ (r & 7)) << 4);
        float sp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (MODE == kBandMerge && so_ok) bf16x8_to_f32(*reinterpret_cast<const uint4*>(sbase + L::kK + off), sp);
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // out = O / l_rnd * w_l + skip partial * w_p, in packed pairs
          float a0, a1;
          f2unpack(f2fma(f2pack(o[cl * 8 + 2 * e], o[cl * 8 + 2 * e + 1]), ow2,
                         f2mul(f2pack(sp[2 * e], sp[2 * e + 1]), wp2)),
                   a0, a1);
          __nv_bfloat162 b2 = __floats2bfloat162_rn(a0, a1);
          w[e] = *reinterpret_cast<uint32_t*>(&b2);
        }
        *reinterpret_cast<uint4*>(sbase + L::kV + off) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      // for the backward: D = dout . out over the fp32 output row (the values rounded to bf16 above)
      if (MODE != kResidue && prm.dout && row_ok) {
        const float ow = inv * wl;
        float dsum = 0.f;
#pragma unroll
        for (int cl = 0; cl < D / 8; ++cl) {
          float g[8], sp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(prm.dout + orow * D + cl * 8), g);
          if (MODE == kBandMerge && so_ok) {
            const uint32_t off = (cl >> 3) * (BM * 128) + r * 128 + (((cl & 7) ^ (r & 7)) << 4);
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(sbase + L::kK + off), sp);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) dsum = fmaf(fmaf(o[cl * 8 + e], ow, sp[e] * wp), g[e], dsum);
        }
        prm.Dout[orow] = dsum;
      }
      lse_log2 = lse2;
      fence_proxy_async_smem();
    }
    // Every softmax warp passes this barrier, epilogue or not (a warp that gave up on a wait must
    // not leave the others blocked here); the tile is then staged whenever it is stored.
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (have_o || no_keys) {
      if (threadIdx.x == 64) {
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          if (MODE == kResidue)
            tma_store_4d(&tmo, sV + c * BM * 128, c * 64, res, (int)q0, bh);
          else
            tma_store_3d(&tmo, sV + c * BM * 128, c * 64, (int)q0, bh);
        }
        tma_store_commit_and_wait_read();  // shared memory must outlive the reads of the store
      }
      if (row_ok) {
        // a row with no key in this pass (only possible for kResidue) has lse -inf
        const float lse2 = lse_log2;
        const float lse_val = l_sum > 0.f ? lse2 * kLn2 : NEG_INF;
        if (MODE == kResidue) prm.skip_lse[orow] = lse_val;
        else if (prm.lse) prm.lse[orow] = lse_val;
        if (MODE != kResidue && prm.lse2) {
          prm.lse2[orow] = lse_val * kLog2e;
          prm.bl2[orow] = bias_l;
          prm.bp2[orow] = bias_p;
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

// ---- host side --------------------------------------------------------------------------------------
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [B*H, n, d] bf16 as a 3-D tensor (d innermost); box = 64 elements x 128 rows x 1.
inline bool make_map(CUtensorMap* m, const void* ptr, int BH, int n, int d, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)n * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The residue-class view of [B*H, n, d] with n = T*pi: a 4-D tensor (d, residue, t, bh) in which
// row t of residue r is sequence row t*pi + r; box = 64 elements x 1 residue x box_rows rows x 1.
inline bool make_residue_map(CUtensorMap* m, const void* ptr, int BH, int n, int d, int pi, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)pi, (cuuint64_t)(n / pi), (cuuint64_t)BH};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)pi * d * 2, (cuuint64_t)n * d * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int MODE>
cudaError_t set_smem_attr() {
  static bool done = false;
  if (done) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel<D, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Smem<D>::kAlloc);
  if (e == cudaSuccess) done = true;
  return e;
}

}  // namespace tc

inline bool tc_supported(bool bf16, int d, int n) { return bf16 && (d == 64 || d == 128) && n >= 1; }

// The backward's split (residue passes + window passes) applies when the sequence is a whole number
// of periods (the residue view is a plain 4-D tensor) and the residue sequences fit the int
// coordinates.
inline bool tc_split_applies(int n, int kwin, int pi, int S) {
  const int m0 = first_skip_m(kwin, pi);
  return S >= m0 && n % pi == 0 && (long long)pi * ((n / pi + tc::BM - 1) / tc::BM) < 0x7fffffffLL;
}

// The forward's split applies from one whole period on: the residue view covers the whole
// periods, rows [0, (n / pi) pi), and the query tiles that reach past them run the single pass.
inline bool tc_split_applies_fwd(int n, int kwin, int pi, int S) {
  const int m0 = first_skip_m(kwin, pi);
  return S >= m0 && n >= pi && (long long)pi * ((n / pi + tc::BM - 1) / tc::BM) < 0x7fffffffLL;
}

// Query tiles of the forward's split path: [0, tiles_merge) take the band-merge pass (every one of
// their rows has a skip partial from the residue pass), the rest the single pass.
inline int split_merge_tiles(int n, int pi) {
  const long long whole = (long long)(n / pi) * pi;  // rows covered by the residue view
  const int tiles = (n + tc::BM - 1) / tc::BM;
  return whole == n ? tiles : (int)(whole / tc::BM);
}

// Pick the split when the skips would cost more tensor work as diagonal tiles than the extra
// HBM traffic of the split costs: diagonal skip tiles ~ S' per query tile vs ~(k + 128)/128 window
// tiles; the split adds ~1.3 KB of traffic per row.
// The bidirectional forward's split: the forward skips of a row may reach past the whole periods,
// so the residue view must hold every row (n a whole number of periods, as the backward's).
inline bool tc_split_applies_bidir(int n, int kwin, int pi, int S) { return tc_split_applies(n, kwin, pi, S); }

inline bool tc_split_preferred(int n, int kwin, int pi, int S, bool fwd = false, bool bidir = false) {
  if (!(bidir ? tc_split_applies_bidir(n, kwin, pi, S)
              : fwd ? tc_split_applies_fwd(n, kwin, pi, S) : tc_split_applies(n, kwin, pi, S)))
    return false;
  const int m0 = first_skip_m(kwin, pi);
  const int nskip = S - m0 + 1;
  const int band_tiles = (kwin + 127) / 128 + 1;
  return pi >= tc::BN && nskip > 2 * band_tiles;
}

// A shard takes the split path where a whole sequence of its length would, and its rows and its
// k/v rows start on whole periods (the residue views of its buffers align with the sequence's).
inline bool shard_split_applies(int n_q, long long row0, long long kv0, int kwin, int pi, int S) {
  return row0 % pi == 0 && kv0 % pi == 0 && tc_split_preferred(n_q, kwin, pi, S, true, false);
}

template <int D>
cudaError_t launch_fwd_tc_d(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                            void* out, float* lse, int B, int H, int n, int kwin, int pi, int S, bool split,
                            bool bidir, void* workspace, cudaStream_t st, const char** why,
                            const void* dout = nullptr, float* Dout = nullptr, float* lse2 = nullptr,
                            float* bl2 = nullptr, float* bp2 = nullptr, long long row0 = 0, long long kv0 = 0,
                            int n_kv = 0) {
  // A shard (row0, kv0, n_kv given): q and out hold sequence rows row0 .., k and v the n_kv
  // sequence rows kv0 ..; the split needs row0 and kv0 on whole periods (the residue views of the
  // two buffers then align).  Otherwise k and v hold the same n rows as q.
  using L = tc::Smem<D>;
  CUtensorMap mq, mk, mv;
  const int BH = B * H;
  if (n_kv <= 0) n_kv = n;
  if (!tc::make_map(&mq, q, BH, n, D, tc::BM) || !tc::make_map(&mk, k, BH, n_kv, D, tc::BN) ||
      !tc::make_map(&mv, v, BH, n_kv, D, tc::BN)) {
    *why = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  tc::Params p;
  p.w_g = w_g;
  p.b_g = b_g;
  p.out = (__nv_bfloat16*)out;
  p.lse = lse;
  p.skip_o = nullptr;
  p.skip_lse = nullptr;
  p.H = H;
  p.n = n;
  p.kwin = kwin;
  p.pi = pi;
  p.S = S;
  p.T = n / pi;
  p.scale_log2 = (float)(1.0 / std::sqrt((double)D)) * kLog2e;
  p.bidir = bidir ? 1 : 0;
  p.tile0 = 0;
  p.row0 = row0;
  p.kv0 = kv0;
  p.dout = (const __nv_bfloat16*)dout;
  p.Dout = Dout;
  p.lse2 = lse2;
  p.bl2 = bl2;
  p.bp2 = bp2;
  const dim3 grid((unsigned)((n + tc::BM - 1) / tc::BM), (unsigned)BH);
  cudaError_t e;
  CUtensorMap mo;
  if (!tc::make_map(&mo, out, BH, n, D, tc::BM)) {
    *why = "cuTensorMapEncodeTiled (out) failed";
    return cudaErrorInvalidValue;
  }
  if (!split) {
    if ((e = tc::set_smem_attr<D, tc::kFused>()) != cudaSuccess) { *why = "cudaFuncSetAttribute"; return e; }
    tc::fwd_tc_kernel<D, tc::kFused><<<grid, tc::kThreads, L::kAlloc, st>>>(mq, mk, mv, mo, mo, p);
    *why = "tensor-core kernel launch";
    return cudaGetLastError();
  }
  CUtensorMap rq, rk, rv;
  if (!tc::make_residue_map(&rq, q, BH, n, D, pi, tc::BM) || !tc::make_residue_map(&rk, k, BH, n_kv, D, pi, tc::BN) ||
      !tc::make_residue_map(&rv, v, BH, n_kv, D, pi, tc::BN)) {
    *why = "cuTensorMapEncodeTiled (residue view) failed";
    return cudaErrorInvalidValue;
  }
  if ((e = tc::set_smem_attr<D, tc::kResidue>()) != cudaSuccess) { *why = "cudaFuncSetAttribute"; return e; }
  if ((e = tc::set_smem_attr<D, tc::kBandMerge>()) != cudaSuccess) { *why = "cudaFuncSetAttribute"; return e; }
  // scratch for the skip partials: [B*H, n, D] bf16 + [B*H, n] fp32 -- the caller's workspace,
  // else taken from cudaMallocAsync on the stream and given back after the second launch
  const size_t rows = (size_t)BH * n;
  void* scratch = workspace;
  const bool own = scratch == nullptr;
  if (own && (e = cudaMallocAsync(&scratch, rows * (D * 2 + 4), st)) != cudaSuccess) {
    *why = "skip-partial scratch allocation";
    return e;
  }
  p.skip_o = (__nv_bfloat16*)scratch;
  p.skip_lse = (float*)((char*)scratch + rows * D * 2);
  CUtensorMap rso, mso;  // the skip partials, in the residue view (stored) and the sequence view (loaded)
  if (!tc::make_residue_map(&rso, p.skip_o, BH, n, D, pi, tc::BM) || !tc::make_map(&mso, p.skip_o, BH, n, D, tc::BM)) {
    if (own) cudaFreeAsync(scratch, st);
    *why = "cuTensorMapEncodeTiled (skip partials) failed";
    return cudaErrorInvalidValue;
  }
  const dim3 grid_r((unsigned)(pi * ((p.T + tc::BM - 1) / tc::BM)), (unsigned)BH);
  tc::fwd_tc_kernel<D, tc::kResidue><<<grid_r, tc::kThreads, L::kAlloc, st>>>(rq, rk, rv, rso, rso, p);
  e = cudaGetLastError();
  // the band-merge pass over the query tiles inside the whole periods; the single pass over the
  // tiles that reach the rows past them (their skips as key tiles, as the fused path takes them)
  const int ntiles = (n + tc::BM - 1) / tc::BM, nmerge = split_merge_tiles(n, pi);
  if (e == cudaSuccess && nmerge > 0) {
    tc::fwd_tc_kernel<D, tc::kBandMerge><<<dim3((unsigned)nmerge, (unsigned)BH), tc::kThreads, L::kAlloc, st>>>(
        mq, mk, mv, mo, mso, p);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess && nmerge < ntiles) {
    if ((e = tc::set_smem_attr<D, tc::kFused>()) == cudaSuccess) {
      tc::Params pt = p;
      pt.tile0 = nmerge;
      tc::fwd_tc_kernel<D, tc::kFused><<<dim3((unsigned)(ntiles - nmerge), (unsigned)BH), tc::kThreads, L::kAlloc,
                                         st>>>(mq, mk, mv, mo, mo, pt);
      e = cudaGetLastError();
    }
  }
  cudaError_t e2 = own ? cudaFreeAsync(scratch, st) : cudaSuccess;
  *why = "tensor-core split kernels";
  return e != cudaSuccess ? e : e2;
}

// One shard of a causal sequence, single pass: q, out [BH, n_q, D] are sequence rows
// row0 .. row0 + n_q - 1; k, v [BH, n_kv, D] are sequence rows kv0 .. kv0 + n_kv - 1 (the halo
// before row0, then the shard's own rows).  The caller has checked that the k/v rows cover every
// key the shard's rows read.
template <int D>
cudaError_t launch_fwd_tc_shard_d(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                                  void* out, float* lse, int B, int H, int n_q, int n_kv, long long row0,
                                  long long kv0, int kwin, int pi, int S, cudaStream_t st, const char** why) {
  using L = tc::Smem<D>;
  CUtensorMap mq, mk, mv, mo;
  const int BH = B * H;
  if (!tc::make_map(&mq, q, BH, n_q, D, tc::BM) || !tc::make_map(&mk, k, BH, n_kv, D, tc::BN) ||
      !tc::make_map(&mv, v, BH, n_kv, D, tc::BN) || !tc::make_map(&mo, out, BH, n_q, D, tc::BM)) {
    *why = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  tc::Params p;
  p.w_g = w_g;
  p.b_g = b_g;
  p.out = (__nv_bfloat16*)out;
  p.lse = lse;
  p.skip_o = nullptr;
  p.skip_lse = nullptr;
  p.H = H;
  p.n = n_q;
  p.kwin = kwin;
  p.pi = pi;
  p.S = S;
  p.T = 0;
  p.scale_log2 = (float)(1.0 / std::sqrt((double)D)) * kLog2e;
  p.bidir = 0;
  p.tile0 = 0;
  p.row0 = row0;
  p.kv0 = kv0;
  p.dout = nullptr;
  p.Dout = nullptr;
  p.lse2 = p.bl2 = p.bp2 = nullptr;
  cudaError_t e;
  if (shard_split_applies(n_q, row0, kv0, kwin, pi, S))  // the residue pass and the window pass, as the whole
    return launch_fwd_tc_d<D>(q, k, v, w_g, b_g, out, lse, B, H, n_q, kwin, pi, S, true, false, nullptr, st, why,
                              nullptr, nullptr, nullptr, nullptr, nullptr, row0, kv0, n_kv);
  if ((e = tc::set_smem_attr<D, tc::kFused>()) != cudaSuccess) { *why = "cudaFuncSetAttribute"; return e; }
  const dim3 grid((unsigned)((n_q + tc::BM - 1) / tc::BM), (unsigned)BH);
  tc::fwd_tc_kernel<D, tc::kFused><<<grid, tc::kThreads, L::kAlloc, st>>>(mq, mk, mv, mo, mo, p);
  *why = "tensor-core shard kernel launch";
  return cudaGetLastError();
}

// The backward's forward over a whole sequence, writing out, lse and, from the fp32 output rows,
// D = dout . out of every row: the single pass, or (split) the residue pass and the window pass,
// whose skip partials take rows * (2 D + 4) bytes of `workspace` (16-byte aligned).
template <int D>
cudaError_t launch_fwd_tc_with_dot(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                                   const void* dout, void* out, float* lse, float* Dout, float* lse2, float* bl2,
                                   float* bp2, int B, int H, int n, int kwin, int pi, int S, bool bidir, bool split,
                                   void* workspace, cudaStream_t st, const char** why) {
  return launch_fwd_tc_d<D>(q, k, v, w_g, b_g, out, lse, B, H, n, kwin, pi, S, split, bidir, workspace, st, why, dout,
                            Dout, lse2, bl2, bp2);
}

// mode: 0 = choose, 1 = single pass, 2 = split (residue pass + window pass)
inline cudaError_t launch_fwd_tc(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                                 void* out, float* lse, int B, int H, int n, int d, int kwin, int pi, int S, int mode,
                                 bool bidir, void* workspace, cudaStream_t st, const char** why) {
  const bool split = mode == 2 || (mode == 0 && tc_split_preferred(n, kwin, pi, S, true, bidir));
  if (d == 128)
    return launch_fwd_tc_d<128>(q, k, v, w_g, b_g, out, lse, B, H, n, kwin, pi, S, split, bidir, workspace, st, why);
  return launch_fwd_tc_d<64>(q, k, v, w_g, b_g, out, lse, B, H, n, kwin, pi, S, split, bidir, workspace, st, why);
}

}  // namespace pia
