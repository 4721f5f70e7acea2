// pi_attn.cu -- the C ABI (include/pi_attn.h): argument checks, kernel choice and launches.
//
// One translation unit holds every kernel so that they share the device error word.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/pi_attn.h"
#include "common.cuh"
#include "bwd_simt.cuh"
#include "decode.cuh"
#include "fwd_simt.cuh"
#include "fwd_tc.cuh"
#include "bwd_tc.cuh"

namespace {

thread_local char g_msg[512] = "";

pi_attn_status fail(pi_attn_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return st;
}

pi_attn_status ok() {
  g_msg[0] = 0;
  return PI_ATTN_OK;
}

pi_attn_status cuda_fail(cudaError_t e, const char* what) {
  return fail(PI_ATTN_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(pi_attn_dtype dt) { return dt == PI_ATTN_BF16 ? 2 : 4; }

// Checks shared by prefill and decode.  n_kv is the sequence (prefill) or cache (decode) length.
pi_attn_status check_common(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                            const void* out, int B, int H, int n_kv, int d, int k_win, int pi, int S,
                            pi_attn_dtype dtype) {
  if (!q || !k || !v || !w_g || !b_g || !out) return fail(PI_ATTN_EINVAL, "null tensor pointer");
  if (dtype != PI_ATTN_F32 && dtype != PI_ATTN_BF16) return fail(PI_ATTN_EINVAL, "unknown dtype %d", (int)dtype);
  if (B < 1 || H < 1 || n_kv < 1) return fail(PI_ATTN_EINVAL, "B, H and n must be >= 1 (got %d, %d, %d)", B, H, n_kv);
  if (d < 1 || d > 256) return fail(PI_ATTN_EINVAL, "d must be in [1, 256] (got %d)", d);
  if ((d * (int)elem_size(dtype)) % 16 != 0)
    return fail(PI_ATTN_EINVAL, "d * sizeof(dtype) must be a multiple of 16 bytes (d = %d)", d);
  if (k_win < 0 || pi < 1 || S < 0) return fail(PI_ATTN_EINVAL, "need k_win >= 0, pi >= 1, S >= 0");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(PI_ATTN_EINVAL, "q, k, v and out must be 16-byte aligned");
  const long long total = (long long)B * H * n_kv * d;
  if (total / d / n_kv / H != B) return fail(PI_ATTN_EINVAL, "tensor size overflows");
  return PI_ATTN_OK;
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// ---- scratch that needs no allocation (pi_attn_decode_noalloc) ----------------------------------
// A fixed device array, part of the library image: every GPU that loads the library holds it
// until the process exits.  Host code must not pass its name to a kernel (on the host the name is
// only a stand-in for the symbol); the device address comes from cudaGetSymbolAddress, once per
// device, with that device current.
constexpr size_t kNoAllocScratchFloats = (size_t)1 << 20;  // 4 MiB
__device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on first use per device).
cudaError_t noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = static_cast<float*>(ptr);
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

// ---- a second stream per device (the tensor-core backward's dk/dv passes beside its dq passes) ---
// Created on first use per device: a non-blocking stream and two events without timing.  A call
// forks onto it and joins back with the lock held, so that calls from several host threads do not
// record over each other's events between a record and its wait; the kernels themselves run
// outside the lock.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_side_mu;
SideStream g_side[kMaxDevices];

cudaError_t side_stream(SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_side_mu);
  SideStream& ss = g_side[dev];
  if (!ss.stream) {
    cudaStream_t st = nullptr;
    cudaEvent_t f = nullptr, j = nullptr;
    if ((e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&f, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&j, cudaEventDisableTiming)) != cudaSuccess) {
      if (f) cudaEventDestroy(f);
      cudaStreamDestroy(st);
      return e;
    }
    ss.stream = st;
    ss.fork = f;
    ss.join = j;
  }
  *out = &ss;
  return cudaSuccess;
}

// Work on `side` after everything enqueued on `s` so far.
cudaError_t side_fork(SideStream& ss, cudaStream_t s) {
  std::lock_guard<std::mutex> lock(g_side_mu);
  cudaError_t e = cudaEventRecord(ss.fork, s);
  return e == cudaSuccess ? cudaStreamWaitEvent(ss.stream, ss.fork, 0) : e;
}
// Work on `s` after everything enqueued on `side` so far.
cudaError_t side_join(SideStream& ss, cudaStream_t s) {
  std::lock_guard<std::mutex> lock(g_side_mu);
  cudaError_t e = cudaEventRecord(ss.join, ss.stream);
  return e == cudaSuccess ? cudaStreamWaitEvent(s, ss.join, 0) : e;
}

// ---- the host-buffer entry points' copy streams (pi_attn_fwd_host, pi_attn_bwd_host) ------------------
// Per device: a stream for the copies in, one for the copies out, and events for the three
// rotating chunk buffers of the workspace (loaded, computed, free again) plus two for the joins.
// A call holds the lock for its whole enqueue sequence: its events are recorded and waited on in
// one order, whatever other host threads do.
constexpr int kHostSets = 3;
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, join_in = nullptr, join_out = nullptr;
  cudaEvent_t loaded[kHostSets] = {}, computed[kHostSets] = {}, freed[kHostSets] = {};
};
std::mutex g_pipe_mu;
HostPipe g_pipe[kMaxDevices];

// The current device's pipe, created on first use; call with g_pipe_mu held.
cudaError_t host_pipe(HostPipe** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  HostPipe& hp = g_pipe[dev];
  if (!hp.in) {
    HostPipe t;
    e = cudaStreamCreateWithFlags(&t.in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&t.out, cudaStreamNonBlocking);
    cudaEvent_t* evs[] = {&t.start, &t.join_in, &t.join_out, &t.loaded[0], &t.loaded[1], &t.loaded[2],
                          &t.computed[0], &t.computed[1], &t.computed[2], &t.freed[0], &t.freed[1], &t.freed[2]};
    for (cudaEvent_t* ev : evs)
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      for (cudaEvent_t* ev : evs)
        if (*ev) cudaEventDestroy(*ev);
      if (t.in) cudaStreamDestroy(t.in);
      if (t.out) cudaStreamDestroy(t.out);
      return e;
    }
    hp = t;
  }
  *out = &hp;
  return cudaSuccess;
}

long long round256(long long x) { return (x + 255) / 256 * 256; }
// (b, h) heads per chunk of pi_attn_fwd_host: the caller's choice, or about a thirty-second of H
// (on bf16_n128k one-head chunks came closest to the host-to-device copy time: 65.4 ms a step
// against 57.9 ms for the copy alone, 67.0 ms with four heads, 68.7 ms with eight)
int host_chunk_heads(int H, int chunk_heads) {
  if (chunk_heads > 0) return chunk_heads < H ? chunk_heads : H;
  return (H + 31) / 32;
}
// One rotating buffer set: q, k, v and out of a chunk, then its lse.
long long host_set_bytes(int hc, int n, int d, int elem) {
  return 4 * round256((long long)hc * n * d * elem) + round256((long long)hc * n * 4);
}

int num_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <typename T, bool DECODE>
pi_attn_status launch_simt(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                           const int* cache_len, void* out, float* lse, int B, int H, int n_q, int n_kv, int d,
                           int k_win, int pi, int S, cudaStream_t st, bool bidir = false) {
  const long long tasks = DECODE ? (long long)B * H : (long long)B * H * n_q;
  const int warps_per_block = 8;
  const long long blocks = (tasks + warps_per_block - 1) / warps_per_block;
  if (blocks > 0x7fffffffLL) return fail(PI_ATTN_EINVAL, "too many query rows");
  const float scale_log2 = (float)(1.0 / std::sqrt((double)d)) * pia::kLog2e;
  pia::simt_attn_kernel<T, DECODE><<<(unsigned)blocks, warps_per_block * 32, 0, st>>>(
      (const T*)q, (const T*)k, (const T*)v, w_g, b_g, cache_len, (T*)out, lse, B, H, n_q, n_kv, d, k_win, pi, S,
      scale_log2, bidir);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ok() : cuda_fail(e, "simt kernel launch");
}

// The tiled backward kernels for one element type: the column count per thread is a template
// (d <= 64, 128 or 256); shared memory above 48 KB is opted into once per instantiation.
template <typename T, int CPT>
cudaError_t launch_bwd_cpt(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                           const void* dout, float* dq, float* dk, float* dv, pia::BwdRowStats rs, dim3 grid, int H,
                           int n, int d, int kwin, int pi, int S, float scale_log2, bool bidir, cudaStream_t s) {
  static bool attr_done = false;
  const size_t sr = pia::bwd_row_smem(d, sizeof(T)), sk = pia::bwd_key_smem(d, sizeof(T));
  if (!attr_done) {
    const size_t max_r = pia::bwd_row_smem(8 * CPT, sizeof(T)), max_k = pia::bwd_key_smem(8 * CPT, sizeof(T));
    cudaError_t e = cudaFuncSetAttribute(pia::bwd_row_kernel<T, CPT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)max_r);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(pia::bwd_key_kernel<T, CPT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)max_k);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  pia::bwd_row_kernel<T, CPT><<<grid, pia::kBwdThreads, sr, s>>>((const T*)q, (const T*)k, (const T*)v, w_g, b_g,
                                                                 (const T*)dout, dq, rs, H, n, d, kwin, pi, S,
                                                                 scale_log2, bidir);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pia::bwd_key_kernel<T, CPT><<<grid, pia::kBwdThreads, sk, s>>>((const T*)q, (const T*)k, (const T*)v,
                                                                 (const T*)dout, rs, dk, dv, H, n, d, kwin, pi, S,
                                                                 scale_log2, bidir);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_bwd(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                       const void* dout, float* dq, float* dk, float* dv, pia::BwdRowStats rs, dim3 grid, int H, int n,
                       int d, int kwin, int pi, int S, float scale_log2, bool bidir, cudaStream_t s) {
  if (d <= 64)
    return launch_bwd_cpt<T, 8>(q, k, v, w_g, b_g, dout, dq, dk, dv, rs, grid, H, n, d, kwin, pi, S, scale_log2, bidir, s);
  if (d <= 128)
    return launch_bwd_cpt<T, 16>(q, k, v, w_g, b_g, dout, dq, dk, dv, rs, grid, H, n, d, kwin, pi, S, scale_log2, bidir,
                                 s);
  return launch_bwd_cpt<T, 32>(q, k, v, w_g, b_g, dout, dq, dk, dv, rs, grid, H, n, d, kwin, pi, S, scale_log2, bidir,
                               s);
}

static long long gate_chunks(int B, int n) {
  return ((long long)B * n + pia::kGateRows - 1) / pia::kGateRows;
}

// Backward scratch: lse2, D, two log2-priors and dz per query row, then the gate's per-chunk
// partial sums (fp32); the tensor-core path adds, 16-byte aligned, the forward's out (bf16) and
// lse (fp32) of every row.
// The tensor-core dq pass writes one gate partial per (b, 128-row query tile).
static long long tc_gate_chunks(int B, int n) { return (long long)B * ((n + pia::tc::BM - 1) / pia::tc::BM); }

static long long bwd_ws_bytes(int B, int H, int n, int d, bool tc) {
  if (B < 1 || H < 1 || n < 1 || d < 1) return 0;
  const long long chunks = tc ? tc_gate_chunks(B, n) : gate_chunks(B, n);
  const long long base = 4LL * (5LL * B * H * n + (long long)H * chunks * (d + 1));
  if (!tc) return base;
  const long long rows = (long long)B * H * n;
  return (base + 15) / 16 * 16 + rows * 2LL * d + rows * 4LL;
}

// Decode: how many CTAs share one (b, h).  Split only when there are too few (b, h) to fill the
// GPU (two-warp CTAs, ~14 resident per SM), keeping >= 128 cache rows per split, at most 64.
int decode_splits(long long bh, int k_win, int S) {
  const long long rows = (long long)k_win + 1 + S;
  const long long slots = 14LL * num_sms();
  if (bh * 2 >= slots) return 1;
  long long ns = (slots + bh - 1) / bh;
  const long long max_ns = (rows + 127) / 128;
  if (ns > max_ns) ns = max_ns;
  if (ns > 64) ns = 64;
  return ns < 1 ? 1 : (int)ns;
}

// Floats of split workspace a decode with these sizes needs (0 without a split).
size_t decode_part_floats(long long bh, int nsplit, int d) { return nsplit > 1 ? (size_t)bh * nsplit * (d + 2) : 0; }

// The decode kernel (and, with a split, the combine kernel) on a filled DecodeArgs whose `part`
// points at decode_part_floats(...) floats of workspace when nsplit > 1.
cudaError_t launch_decode(const pia::DecodeArgs& a, int d, long long bh, cudaStream_t s) {
  dim3 grid((unsigned)bh, (unsigned)a.nsplit);
  if (d == 128) pia::decode_bf16_kernel<128><<<grid, 64, 0, s>>>(a);
  else pia::decode_bf16_kernel<64><<<grid, 64, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && a.nsplit > 1) {
    if (d == 128)
      pia::decode_combine_kernel<128><<<(unsigned)bh, 128, 0, s>>>(a.part, a.nsplit, a.cache_len, a.H, a.n_cache,
                                                                  a.out, a.lse, a.ring);
    else
      pia::decode_combine_kernel<64><<<(unsigned)bh, 64, 0, s>>>(a.part, a.nsplit, a.cache_len, a.H, a.n_cache,
                                                                a.out, a.lse, a.ring);
    e = cudaGetLastError();
  }
  return e;
}

// DecodeArgs for a bf16 decode call (no workspace yet).
pia::DecodeArgs decode_args(const void* q, const void* kcache, const void* vcache, const float* w_g, const float* b_g,
                            const int* cache_len, void* out, float* lse, int H, int n_cache, int d, int k_win, int pi,
                            int S, int nsplit, bool ring) {
  pia::DecodeArgs a;
  a.q = (const __nv_bfloat16*)q;
  a.kc = (const __nv_bfloat16*)kcache;
  a.vc = (const __nv_bfloat16*)vcache;
  a.w_g = w_g;
  a.b_g = b_g;
  a.cache_len = cache_len;
  a.out = (__nv_bfloat16*)out;
  a.lse = lse;
  a.part = nullptr;
  a.H = H;
  a.n_cache = n_cache;
  a.kwin = k_win;
  a.pi = pi;
  a.S = S;
  a.nsplit = nsplit;
  a.scale_log2 = (float)(1.0 / std::sqrt((double)d)) * pia::kLog2e;
  a.ring = ring ? 1 : 0;
  return a;
}

}  // namespace

extern "C" {

const char* pi_attn_status_string(pi_attn_status s) {
  switch (s) {
    case PI_ATTN_OK: return "PI_ATTN_OK";
    case PI_ATTN_EINVAL: return "PI_ATTN_EINVAL";
    case PI_ATTN_EUNSUPPORTED: return "PI_ATTN_EUNSUPPORTED";
    case PI_ATTN_ECUDA: return "PI_ATTN_ECUDA";
    case PI_ATTN_EDEVICE: return "PI_ATTN_EDEVICE";
  }
  return "PI_ATTN_<unknown>";
}

const char* pi_attn_last_error(void) { return g_msg; }

int pi_attn_version(void) { return 100; }

// Which kernels a forward call with these arguments runs: *tc (tensor-core path) and *split
// (residue pass + band-merge pass), after the same checks as the call itself.
// The tensor-core kernels take the (b, h) pairs as their grid's y dimension.
constexpr long long kMaxGridY = 65535;

static pi_attn_status fwd_route(long long bh, int n, int d, int k_win, int pi, int S, pi_attn_dtype dtype,
                                pi_attn_path path, bool bidir, bool* tc, bool* split) {
  if (path < PI_ATTN_PATH_AUTO || path > PI_ATTN_PATH_TC_SPLIT) return fail(PI_ATTN_EINVAL, "unknown path %d", (int)path);
  const bool tc_ok = pia::tc_supported(dtype == PI_ATTN_BF16, d, n) && bh <= kMaxGridY;
  const bool want_tc = path == PI_ATTN_PATH_TC || path == PI_ATTN_PATH_TC_FUSED || path == PI_ATTN_PATH_TC_SPLIT;
  if (want_tc && bh > kMaxGridY)
    return fail(PI_ATTN_EUNSUPPORTED, "tensor-core path takes at most %lld (b, h) pairs a call (got %lld)", kMaxGridY,
                bh);
  if (want_tc && !tc_ok)
    return fail(PI_ATTN_EUNSUPPORTED, "tensor-core path covers bf16 with d in {64, 128} (got dtype %d, d %d)",
                (int)dtype, d);
  if (path == PI_ATTN_PATH_TC_SPLIT && bidir && !pia::tc_split_applies_bidir(n, k_win, pi, S))
    return fail(PI_ATTN_EUNSUPPORTED,
                "the bidirectional split path needs n %% pi == 0 and at least one skip outside the window");
  if (path == PI_ATTN_PATH_TC_SPLIT && !bidir && !pia::tc_split_applies_fwd(n, k_win, pi, S))
    return fail(PI_ATTN_EUNSUPPORTED, "split path needs n >= pi and at least one skip outside the window");
  *tc = path != PI_ATTN_PATH_SIMT && tc_ok;
  *split = *tc && (path == PI_ATTN_PATH_TC_SPLIT ||
                   (path != PI_ATTN_PATH_TC_FUSED && pia::tc_split_preferred(n, k_win, pi, S, true, bidir)));
  return ok();
}

static long long fwd_scratch_bytes(int B, int H, int n, int d, bool split) {
  return split ? (long long)B * H * n * (2LL * d + 4) : 0;
}

static pi_attn_status fwd_impl(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                               void* out, float* lse, int B, int H, int n, int d, int k_win, int pi, int S,
                               pi_attn_dtype dtype, pi_attn_path path, bool bidir, void* workspace,
                               long long workspace_bytes, void* stream) {
  pi_attn_status st = check_common(q, k, v, w_g, b_g, out, B, H, n, d, k_win, pi, S, dtype);
  if (st != PI_ATTN_OK) return st;
  bool tc = false, split = false;
  if ((st = fwd_route((long long)B * H, n, d, k_win, pi, S, dtype, path, bidir, &tc, &split)) != PI_ATTN_OK) return st;
  if (workspace) {
    if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0) return fail(PI_ATTN_EINVAL, "workspace not 16-byte aligned");
    const long long need = fwd_scratch_bytes(B, H, n, d, split);
    if (workspace_bytes < need)
      return fail(PI_ATTN_EINVAL, "workspace of %lld bytes, this call needs %lld", workspace_bytes, need);
  }
  cudaStream_t s = as_stream(stream);
  if (tc) {
    const char* why = nullptr;
    const int mode = split ? 2 : 1;
    cudaError_t e =
        pia::launch_fwd_tc(q, k, v, w_g, b_g, out, lse, B, H, n, d, k_win, pi, S, mode, bidir, workspace, s, &why);
    if (e != cudaSuccess) return cuda_fail(e, why ? why : "tensor-core kernel launch");
    return ok();
  }
  if (dtype == PI_ATTN_F32)
    return launch_simt<float, false>(q, k, v, w_g, b_g, nullptr, out, lse, B, H, n, n, d, k_win, pi, S, s, bidir);
  return launch_simt<__nv_bfloat16, false>(q, k, v, w_g, b_g, nullptr, out, lse, B, H, n, n, d, k_win, pi, S, s,
                                           bidir);
}

pi_attn_status pi_attn_fwd_ws(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                              void* out, float* lse, int B, int H, int n, int d, int k_win, int pi, int S,
                              pi_attn_dtype dtype, pi_attn_path path, void* workspace, long long workspace_bytes,
                              void* stream) {
  return fwd_impl(q, k, v, w_g, b_g, out, lse, B, H, n, d, k_win, pi, S, dtype, path, false, workspace,
                  workspace_bytes, stream);
}

pi_attn_status pi_attn_fwd_bidir(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                                 void* out, float* lse, int B, int H, int n, int d, int k_win, int pi, int S,
                                 pi_attn_dtype dtype, pi_attn_path path, void* stream) {
  return fwd_impl(q, k, v, w_g, b_g, out, lse, B, H, n, d, k_win, pi, S, dtype, path, true, nullptr, 0, stream);
}

long long pi_attn_fwd_shard_scratch_bytes(int B, int H, int n_q, long long row0, long long kv0, int d, int k_win,
                                          int pi, int S) {
  if (B < 1 || H < 1 || n_q < 1 || d < 1 || row0 < 0 || kv0 < 0 || k_win < 0 || pi < 1 || S < 0) return -1;
  return pia::shard_split_applies(n_q, row0, kv0, k_win, pi, S) ? (long long)B * H * n_q * (2LL * d + 4) : 0;
}

pi_attn_status pi_attn_fwd_shard_ws(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                                    void* out, float* lse, int B, int H, int n_q, int n_kv, long long row0,
                                    long long kv0, int d, int k_win, int pi, int S, pi_attn_dtype dtype,
                                    void* workspace, long long workspace_bytes, void* stream) {
  pi_attn_status st = check_common(q, k, v, w_g, b_g, out, B, H, n_kv, d, k_win, pi, S, dtype);
  if (st != PI_ATTN_OK) return st;
  if (n_q < 1) return fail(PI_ATTN_EINVAL, "n_q must be >= 1 (got %d)", n_q);
  if ((long long)B * H * n_q * d / d / n_q / H != B) return fail(PI_ATTN_EINVAL, "tensor size overflows");
  if (dtype != PI_ATTN_BF16 || (d != 64 && d != 128))
    return fail(PI_ATTN_EUNSUPPORTED, "the shard forward covers bf16 with d in {64, 128} (got dtype %d, d %d)",
                (int)dtype, d);
  if (row0 < 0 || kv0 < 0) return fail(PI_ATTN_EINVAL, "row0 and kv0 must be >= 0");
  // every key a shard row reads: the window back to row0 - k_win and the skips back to row0 - S*pi
  // (only those past the window exist), through the shard's last row
  const long long m0 = k_win / pi + 1;
  long long reach = k_win;
  if (S >= m0 && (long long)S * pi > reach) reach = (long long)S * pi;
  const long long need_lo = row0 - reach > 0 ? row0 - reach : 0;
  if (kv0 > need_lo)
    return fail(PI_ATTN_EINVAL, "k/v rows start at %lld, after the first key the shard reads (%lld)", kv0, need_lo);
  if (kv0 + n_kv < row0 + n_q)
    return fail(PI_ATTN_EINVAL, "k/v rows end at %lld, before the shard's last row %lld", kv0 + n_kv - 1,
                row0 + n_q - 1);
  if (row0 + n_q > 0x7fffffffLL) return fail(PI_ATTN_EINVAL, "sequence rows past 2^31");
  if ((long long)B * H > kMaxGridY)
    return fail(PI_ATTN_EUNSUPPORTED, "the shard forward takes at most %lld (b, h) pairs a call (got %lld)", kMaxGridY,
                (long long)B * H);
  // the split path (residue pass, band-merge pass, tail) where the shard's rows and halo start on
  // whole periods, its skip partials in the caller's workspace (else cudaMallocAsync on `stream`)
  const bool split = pia::shard_split_applies(n_q, row0, kv0, k_win, pi, S);
  if (workspace) {
    if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0) return fail(PI_ATTN_EINVAL, "workspace not 16-byte aligned");
    const long long need = split ? (long long)B * H * n_q * (2LL * d + 4) : 0;
    if (workspace_bytes < need)
      return fail(PI_ATTN_EINVAL, "workspace of %lld bytes, the shard needs %lld", workspace_bytes, need);
  }
  const char* why = "";
  const cudaStream_t s = as_stream(stream);
  cudaError_t e;
  if (split)
    e = d == 128 ? pia::launch_fwd_tc_d<128>(q, k, v, w_g, b_g, out, lse, B, H, n_q, k_win, pi, S, true, false,
                                             workspace, s, &why, nullptr, nullptr, nullptr, nullptr, nullptr, row0,
                                             kv0, n_kv)
                 : pia::launch_fwd_tc_d<64>(q, k, v, w_g, b_g, out, lse, B, H, n_q, k_win, pi, S, true, false,
                                            workspace, s, &why, nullptr, nullptr, nullptr, nullptr, nullptr, row0,
                                            kv0, n_kv);
  else
    e = d == 128 ? pia::launch_fwd_tc_shard_d<128>(q, k, v, w_g, b_g, out, lse, B, H, n_q, n_kv, row0, kv0, k_win,
                                                   pi, S, s, &why)
                 : pia::launch_fwd_tc_shard_d<64>(q, k, v, w_g, b_g, out, lse, B, H, n_q, n_kv, row0, kv0, k_win, pi,
                                                  S, s, &why);
  return e == cudaSuccess ? ok() : cuda_fail(e, why);
}

pi_attn_status pi_attn_fwd_shard(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                                 void* out, float* lse, int B, int H, int n_q, int n_kv, long long row0,
                                 long long kv0, int d, int k_win, int pi, int S, pi_attn_dtype dtype, void* stream) {
  return pi_attn_fwd_shard_ws(q, k, v, w_g, b_g, out, lse, B, H, n_q, n_kv, row0, kv0, d, k_win, pi, S, dtype, nullptr,
                              0, stream);
}

pi_attn_status pi_attn_fwd_ex(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                              void* out, float* lse, int B, int H, int n, int d, int k_win, int pi, int S,
                              pi_attn_dtype dtype, pi_attn_path path, void* stream) {
  return pi_attn_fwd_ws(q, k, v, w_g, b_g, out, lse, B, H, n, d, k_win, pi, S, dtype, path, nullptr, 0, stream);
}

long long pi_attn_fwd_host_workspace_bytes(int B, int H, int n, int d, pi_attn_dtype dtype, int chunk_heads) {
  if (B < 1 || H < 1 || n < 1 || d < 1 || chunk_heads < 0 || (dtype != PI_ATTN_F32 && dtype != PI_ATTN_BF16))
    return -1;
  const int hc = host_chunk_heads(H, chunk_heads);
  return kHostSets * host_set_bytes(hc, n, d, (int)elem_size(dtype)) + round256((long long)hc * n * (2LL * d + 4));
}

pi_attn_status pi_attn_fwd_host(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                                void* out, float* lse, int B, int H, int n, int d, int k_win, int pi, int S,
                                pi_attn_dtype dtype, pi_attn_path path, int chunk_heads, void* workspace,
                                long long workspace_bytes, void* stream) {
  if (!q || !k || !v || !out) return fail(PI_ATTN_EINVAL, "null host tensor pointer");
  if (!w_g || !b_g) return fail(PI_ATTN_EINVAL, "null gate parameter pointer");
  if (chunk_heads < 0) return fail(PI_ATTN_EINVAL, "chunk_heads must be >= 0 (got %d)", chunk_heads);
  // the checks every chunk's call makes, once for the whole problem before anything is enqueued
  static const char dummy[16] __attribute__((aligned(16))) = {0};
  pi_attn_status st = check_common(dummy, dummy, dummy, w_g, b_g, dummy, B, H, n, d, k_win, pi, S, dtype);
  if (st != PI_ATTN_OK) return st;
  bool tc = false, split = false;  // (each chunk is a [1, chunk_heads, n, d] problem)
  if ((st = fwd_route(host_chunk_heads(H, chunk_heads), n, d, k_win, pi, S, dtype, path, false, &tc, &split)) !=
      PI_ATTN_OK)
    return st;
  const long long need = pi_attn_fwd_host_workspace_bytes(B, H, n, d, dtype, chunk_heads);
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
    return fail(PI_ATTN_EINVAL, "workspace must be a 256-byte aligned device pointer");
  if (workspace_bytes < need)
    return fail(PI_ATTN_EINVAL, "workspace of %lld bytes, the call needs %lld", workspace_bytes, need);
  const int hc = host_chunk_heads(H, chunk_heads);
  const int elem = (int)elem_size(dtype);
  const long long tile = round256((long long)hc * n * d * elem), set_bytes = host_set_bytes(hc, n, d, elem);
  char* const ws = static_cast<char*>(workspace);
  void* const scratch = ws + kHostSets * set_bytes;
  const long long scratch_bytes = round256((long long)hc * n * (2LL * d + 4));
  cudaStream_t s = as_stream(stream);

  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe* hp = nullptr;
  cudaError_t e = host_pipe(&hp);
  if (e != cudaSuccess) return cuda_fail(e, "copy streams");
  // the copies start after the work already on `stream` (an earlier call may still use the workspace)
  if ((e = cudaEventRecord(hp->start, s)) != cudaSuccess || (e = cudaStreamWaitEvent(hp->in, hp->start, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(hp->out, hp->start, 0)) != cudaSuccess)
    return cuda_fail(e, "copy streams");
  const char* why = "host-buffer chunk copies";
  int c = 0;
  for (int b = 0; b < B && st == PI_ATTN_OK && e == cudaSuccess; ++b) {
    for (int h0 = 0; h0 < H && st == PI_ATTN_OK && e == cudaSuccess; h0 += hc, ++c) {
      const int h = hc < H - h0 ? hc : H - h0, set = c % kHostSets;
      char* const base = ws + set * set_bytes;
      void *dq = base, *dk = base + tile, *dv = base + 2 * tile, *dout = base + 3 * tile;
      float* const dlse = reinterpret_cast<float*>(base + 4 * tile);
      const long long row0 = (long long)b * H + h0;  // first (b, h) of the chunk
      const size_t bytes = (size_t)h * n * d * elem, off = (size_t)row0 * n * d * elem;
      // in: the set's buffers are free once the copies out of the chunk three before have run
      if (c >= kHostSets && (e = cudaStreamWaitEvent(hp->in, hp->freed[set], 0)) != cudaSuccess) break;
      if ((e = cudaMemcpyAsync(dq, static_cast<const char*>(q) + off, bytes, cudaMemcpyHostToDevice, hp->in)) != cudaSuccess ||
          (e = cudaMemcpyAsync(dk, static_cast<const char*>(k) + off, bytes, cudaMemcpyHostToDevice, hp->in)) != cudaSuccess ||
          (e = cudaMemcpyAsync(dv, static_cast<const char*>(v) + off, bytes, cudaMemcpyHostToDevice, hp->in)) != cudaSuccess ||
          (e = cudaEventRecord(hp->loaded[set], hp->in)) != cudaSuccess ||
          (e = cudaStreamWaitEvent(s, hp->loaded[set], 0)) != cudaSuccess)
        break;
      // compute on `stream`: the chunk as a [1, h, n, d] problem with its heads' gate parameters
      st = fwd_impl(dq, dk, dv, w_g + (long long)h0 * d, b_g + h0, dout, lse ? dlse : nullptr, 1, h, n, d, k_win, pi,
                    S, dtype, path, false, scratch, scratch_bytes, stream);
      if (st != PI_ATTN_OK) break;
      // out
      if ((e = cudaEventRecord(hp->computed[set], s)) != cudaSuccess ||
          (e = cudaStreamWaitEvent(hp->out, hp->computed[set], 0)) != cudaSuccess ||
          (e = cudaMemcpyAsync(static_cast<char*>(out) + off, dout, bytes, cudaMemcpyDeviceToHost, hp->out)) != cudaSuccess)
        break;
      if (lse && (e = cudaMemcpyAsync(lse + row0 * n, dlse, (size_t)h * n * 4, cudaMemcpyDeviceToHost, hp->out)) != cudaSuccess)
        break;
      if ((e = cudaEventRecord(hp->freed[set], hp->out)) != cudaSuccess) break;
    }
  }
  // join both copy streams back into `stream`, whatever failed above: the caller's next work on
  // `stream` (and the workspace's next user) must come after every copy this call enqueued
  cudaError_t ej = cudaEventRecord(hp->join_in, hp->in);
  if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, hp->join_in, 0);
  if (ej == cudaSuccess) ej = cudaEventRecord(hp->join_out, hp->out);
  if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, hp->join_out, 0);
  if (st != PI_ATTN_OK) return st;
  if (e != cudaSuccess) return cuda_fail(e, why);
  if (ej != cudaSuccess) return cuda_fail(ej, "joining the copy streams");
  return ok();
}

pi_attn_status pi_attn_fwd_plan(int B, int H, int n, int d, int k_win, int pi, int S, pi_attn_dtype dtype,
                                pi_attn_path path, int* launches, long long* scratch_bytes) {
  static const char dummy[16] __attribute__((aligned(16))) = {0};
  if (!launches || !scratch_bytes) return fail(PI_ATTN_EINVAL, "null output pointer");
  pi_attn_status st = check_common(dummy, dummy, dummy, (const float*)dummy, (const float*)dummy, dummy, B, H, n, d,
                                   k_win, pi, S, dtype);
  if (st != PI_ATTN_OK) return st;
  bool tc = false, split = false;
  if ((st = fwd_route((long long)B * H, n, d, k_win, pi, S, dtype, path, false, &tc, &split)) != PI_ATTN_OK) return st;
  if (split) {  // the residue pass; the band-merge pass and / or the single pass over the ragged tail
    const int ntiles = (n + pia::tc::BM - 1) / pia::tc::BM, nmerge = pia::split_merge_tiles(n, pi);
    *launches = 1 + (nmerge > 0 ? 1 : 0) + (nmerge < ntiles ? 1 : 0);
  } else {
    *launches = 1;
  }
  *scratch_bytes = fwd_scratch_bytes(B, H, n, d, split);
  return ok();
}

pi_attn_status pi_attn_fwd(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                           void* out, float* lse, int B, int H, int n, int d, int k_win, int pi, int S,
                           pi_attn_dtype dtype, void* stream) {
  return pi_attn_fwd_ex(q, k, v, w_g, b_g, out, lse, B, H, n, d, k_win, pi, S, dtype, PI_ATTN_PATH_AUTO, stream);
}

static pi_attn_status decode_impl(const void* q, const void* kcache, const void* vcache, const float* w_g,
                                  const float* b_g, const int* cache_len, void* out, float* lse, int B, int H,
                                  int n_cache, int d, int k_win, int pi, int S, pi_attn_dtype dtype, void* stream,
                                  bool ring) {
  pi_attn_status st = check_common(q, kcache, vcache, w_g, b_g, out, B, H, n_cache, d, k_win, pi, S, dtype);
  if (st != PI_ATTN_OK) return st;
  if (ring) {
    if (dtype != PI_ATTN_BF16 || (d != 64 && d != 128))
      return fail(PI_ATTN_EUNSUPPORTED, "the ring-cache decode covers bf16 with d in {64, 128}");
    const long long reach = (long long)S * pi > k_win ? (long long)S * pi : k_win;
    if ((long long)n_cache < reach + 1)
      return fail(PI_ATTN_EINVAL, "ring capacity %d below max(k_win, S*pi) + 1 = %lld", n_cache, reach + 1);
    if (!cache_len) return fail(PI_ATTN_EINVAL, "the ring-cache decode needs cache_len");
  }
  cudaStream_t s = as_stream(stream);
  if (dtype == PI_ATTN_BF16 && (d == 64 || d == 128)) {
    const long long bh = (long long)B * H;
    if (bh > 0x7fffffffLL) return fail(PI_ATTN_EINVAL, "B * H too large");
    pia::DecodeArgs a = decode_args(q, kcache, vcache, w_g, b_g, cache_len, out, lse, H, n_cache, d, k_win, pi, S,
                                    decode_splits(bh, k_win, S), ring);
    const size_t part = decode_part_floats(bh, a.nsplit, d);
    if (part) {
      cudaError_t e = cudaMallocAsync((void**)&a.part, part * sizeof(float), s);
      if (e != cudaSuccess) return cuda_fail(e, "decode workspace allocation");
    }
    cudaError_t e = launch_decode(a, d, bh, s);
    if (a.part) {
      cudaError_t e2 = cudaFreeAsync(a.part, s);
      if (e == cudaSuccess) e = e2;
    }
    return e == cudaSuccess ? ok() : cuda_fail(e, "decode kernel launch");
  }
  if (dtype == PI_ATTN_F32)
    return launch_simt<float, true>(q, kcache, vcache, w_g, b_g, cache_len, out, lse, B, H, 1, n_cache, d, k_win, pi,
                                    S, s);
  return launch_simt<__nv_bfloat16, true>(q, kcache, vcache, w_g, b_g, cache_len, out, lse, B, H, 1, n_cache, d, k_win,
                                          pi, S, s);
}

pi_attn_status pi_attn_decode(const void* q, const void* kcache, const void* vcache, const float* w_g,
                              const float* b_g, const int* cache_len, void* out, float* lse, int B, int H,
                              int n_cache, int d, int k_win, int pi, int S, pi_attn_dtype dtype, void* stream) {
  return decode_impl(q, kcache, vcache, w_g, b_g, cache_len, out, lse, B, H, n_cache, d, k_win, pi, S, dtype, stream,
                     false);
}

pi_attn_status pi_attn_decode_ring(const void* q, const void* kcache, const void* vcache, const float* w_g,
                                   const float* b_g, const int* cache_len, void* out, float* lse, int B, int H,
                                   int capacity, int d, int k_win, int pi, int S, pi_attn_dtype dtype, void* stream) {
  return decode_impl(q, kcache, vcache, w_g, b_g, cache_len, out, lse, B, H, capacity, d, k_win, pi, S, dtype, stream,
                     true);
}

pi_attn_status pi_attn_cache_append(void* kcache, void* vcache, const void* k_new, const void* v_new, int* cache_len,
                                    int B, int H, int capacity, int d, pi_attn_dtype dtype, int ring, void* stream) {
  if (!kcache || !vcache || !k_new || !v_new || !cache_len) return fail(PI_ATTN_EINVAL, "null pointer");
  if (dtype != PI_ATTN_F32 && dtype != PI_ATTN_BF16) return fail(PI_ATTN_EINVAL, "unknown dtype %d", (int)dtype);
  if (B < 1 || H < 1 || capacity < 1 || d < 1 || d > 256) return fail(PI_ATTN_EINVAL, "bad sizes");
  if ((d * (int)elem_size(dtype)) % 16 != 0) return fail(PI_ATTN_EINVAL, "d * sizeof(dtype) must be a multiple of 16");
  if (!aligned16(kcache) || !aligned16(vcache) || !aligned16(k_new) || !aligned16(v_new))
    return fail(PI_ATTN_EINVAL, "caches and new rows must be 16-byte aligned");
  const long long bh = (long long)B * H;
  if (bh > 0x7fffffffLL) return fail(PI_ATTN_EINVAL, "B * H too large");
  cudaStream_t s = as_stream(stream);
  if (dtype == PI_ATTN_BF16)
    pia::cache_append_kernel<__nv_bfloat16><<<(unsigned)bh, 32, 0, s>>>(
        (__nv_bfloat16*)kcache, (__nv_bfloat16*)vcache, (const __nv_bfloat16*)k_new, (const __nv_bfloat16*)v_new,
        cache_len, H, capacity, d, ring);
  else
    pia::cache_append_kernel<float><<<(unsigned)bh, 32, 0, s>>>((float*)kcache, (float*)vcache, (const float*)k_new,
                                                                (const float*)v_new, cache_len, H, capacity, d, ring);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    pia::cache_len_advance_kernel<<<(B + 255) / 256, 256, 0, s>>>(cache_len, B, capacity, ring);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? ok() : cuda_fail(e, "cache append launch");
}

pi_attn_status pi_attn_decode_noalloc(const void* q, const void* kcache, const void* vcache, const float* w_g,
                                      const float* b_g, const int* cache_len, void* out, float* lse, int B, int H,
                                      int n_cache, int d, int k_win, int pi, int S, pi_attn_dtype dtype,
                                      void* stream) {
  pi_attn_status st = check_common(q, kcache, vcache, w_g, b_g, out, B, H, n_cache, d, k_win, pi, S, dtype);
  if (st != PI_ATTN_OK) return st;
  if (dtype != PI_ATTN_BF16 || (d != 64 && d != 128))
    return fail(PI_ATTN_EUNSUPPORTED, "pi_attn_decode_noalloc covers bf16 with d in {64, 128} (got dtype %d, d %d)",
                (int)dtype, d);
  const long long bh = (long long)B * H;
  if (bh > 0x7fffffffLL) return fail(PI_ATTN_EINVAL, "B * H too large");
  // the same split and the same kernels as pi_attn_decode; only the workspace differs
  pia::DecodeArgs a = decode_args(q, kcache, vcache, w_g, b_g, cache_len, out, lse, H, n_cache, d, k_win, pi, S,
                                  decode_splits(bh, k_win, S), false);
  const size_t need = decode_part_floats(bh, a.nsplit, d);
  if (need > kNoAllocScratchFloats)
    return fail(PI_ATTN_EINVAL,
                "pi_attn_decode_noalloc: %lld (b, h) x %d splits need %zu bytes of scratch, above its fixed %zu",
                bh, a.nsplit, need * sizeof(float), kNoAllocScratchFloats * sizeof(float));
  if (need) {
    cudaError_t e = noalloc_scratch(&a.part);  // every split writes its whole slot: nothing to clear
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(decode scratch)");
  }
  cudaError_t e = launch_decode(a, d, bh, as_stream(stream));
  return e == cudaSuccess ? ok() : cuda_fail(e, "decode kernel launch");
}

static pi_attn_status index_sets_impl(int n, int k_win, int pi, int S, int* counts, int* idx, int width, bool bidir,
                                      void* stream) {
  if (!counts || !idx) return fail(PI_ATTN_EINVAL, "null pointer");
  if (n < 1 || k_win < 0 || pi < 1 || S < 0) return fail(PI_ATTN_EINVAL, "need n >= 1, k_win >= 0, pi >= 1, S >= 0");
  const long long need = bidir ? 2LL * k_win + 1 + 2LL * S : (long long)k_win + 1 + S;
  if ((long long)width < need) return fail(PI_ATTN_EINVAL, "width %d < %lld", width, need);
  const int threads = 256;
  pia::index_sets_kernel<<<(n + threads - 1) / threads, threads, 0, as_stream(stream)>>>(n, k_win, pi, S, width, bidir,
                                                                                          counts, idx);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ok() : cuda_fail(e, "index-set kernel launch");
}

pi_attn_status pi_attn_debug_index_sets(int n, int k_win, int pi, int S, int* counts, int* idx, int width,
                                        void* stream) {
  return index_sets_impl(n, k_win, pi, S, counts, idx, width, false, stream);
}

pi_attn_status pi_attn_debug_index_sets_bidir(int n, int k_win, int pi, int S, int* counts, int* idx, int width,
                                              void* stream) {
  return index_sets_impl(n, k_win, pi, S, counts, idx, width, true, stream);
}

long long pi_attn_bwd_workspace_bytes(int B, int H, int n, int d) { return bwd_ws_bytes(B, H, n, d, false); }

long long pi_attn_bwd_workspace_bytes_ex(int B, int H, int n, int d, pi_attn_dtype dtype, pi_attn_bwd_path path) {
  const bool tc = path == PI_ATTN_BWD_TC || path == PI_ATTN_BWD_TC_FUSED || path == PI_ATTN_BWD_TC_SPLIT ||
                  (path == PI_ATTN_BWD_AUTO && dtype == PI_ATTN_BF16 && (d == 64 || d == 128));
  return bwd_ws_bytes(B, H, n, d, tc);
}

// The backward's kernel choice and the checks it implies, before anything is enqueued.
static pi_attn_status bwd_route(int B, int H, int n, int d, int k_win, int pi, int S, pi_attn_dtype dtype, int bidir,
                                pi_attn_bwd_path path, bool* tc, bool* split) {
  if (path < PI_ATTN_BWD_AUTO || path > PI_ATTN_BWD_TC_SPLIT)
    return fail(PI_ATTN_EINVAL, "unknown backward path %d", (int)path);
  const bool tc_ok = dtype == PI_ATTN_BF16 && (d == 64 || d == 128);
  const bool want_tc = path == PI_ATTN_BWD_TC || path == PI_ATTN_BWD_TC_FUSED || path == PI_ATTN_BWD_TC_SPLIT;
  if (want_tc && !tc_ok)
    return fail(PI_ATTN_EUNSUPPORTED, "the tensor-core backward covers bf16 with d in {64, 128} (got dtype %d, d %d)",
                (int)dtype, d);
  if (path == PI_ATTN_BWD_TC_SPLIT && bidir)
    return fail(PI_ATTN_EUNSUPPORTED, "the split backward covers the causal rule only");
  if (path == PI_ATTN_BWD_TC_SPLIT && !pia::tc_split_applies(n, k_win, pi, S))
    return fail(PI_ATTN_EUNSUPPORTED, "split backward needs n %% pi == 0 and at least one skip outside the window");
  *tc = want_tc || (path == PI_ATTN_BWD_AUTO && tc_ok);
  *split = *tc && !bidir && (path == PI_ATTN_BWD_TC_SPLIT ||
                             (path != PI_ATTN_BWD_TC_FUSED && pia::tc_split_preferred(n, k_win, pi, S)));
  const long long tiles = ((long long)n + pia::kBwdRows - 1) / pia::kBwdRows;
  if (tiles > 0x7fffffffLL || (long long)B * H > 65535) return fail(PI_ATTN_EINVAL, "grid too large");
  const long long nchunks = *tc ? tc_gate_chunks(B, n) : gate_chunks(B, n);
  if (nchunks > 0x7fffffffLL || H > 65535) return fail(PI_ATTN_EINVAL, "too many rows per head for the gate sums");
  return ok();
}

pi_attn_status pi_attn_bwd_ex(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                              const void* dout, float* dq, float* dk, float* dv, float* dw_g, float* db_g, int B,
                              int H, int n, int d, int k_win, int pi, int S, pi_attn_dtype dtype, int bidir,
                              pi_attn_bwd_path path, void* workspace, long long workspace_bytes, void* stream) {
  pi_attn_status st = check_common(q, k, v, w_g, b_g, dout, B, H, n, d, k_win, pi, S, dtype);
  if (st != PI_ATTN_OK) return st;
  if (!dq || !dk || !dv || !dw_g || !db_g) return fail(PI_ATTN_EINVAL, "null gradient pointer");
  if (!aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return fail(PI_ATTN_EINVAL, "dq, dk, dv must be 16-byte aligned");
  bool tc = false, split = false;
  if ((st = bwd_route(B, H, n, d, k_win, pi, S, dtype, bidir, path, &tc, &split)) != PI_ATTN_OK) return st;
  const long long rows = (long long)B * H * n;
  const long long need = bwd_ws_bytes(B, H, n, d, tc);
  if (workspace) {
    if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0) return fail(PI_ATTN_EINVAL, "workspace not 16-byte aligned");
    if (workspace_bytes < need)
      return fail(PI_ATTN_EINVAL, "workspace of %lld bytes, the backward needs %lld", workspace_bytes, need);
  }
  const long long tiles = ((long long)n + pia::kBwdRows - 1) / pia::kBwdRows;
  const long long nchunks = tc ? tc_gate_chunks(B, n) : gate_chunks(B, n);
  cudaStream_t s = as_stream(stream);
  void* scratch = workspace;
  cudaError_t e = cudaSuccess;
  if (!scratch && (e = cudaMallocAsync(&scratch, (size_t)need, s)) != cudaSuccess)
    return cuda_fail(e, "backward scratch allocation");
  float* base = static_cast<float*>(scratch);
  pia::BwdRowStats rs{base, base + rows, base + 2 * rows, base + 3 * rows, base + 4 * rows};
  float* part_w = base + 5 * rows;
  float* part_b = part_w + (long long)H * nchunks * d;
  const dim3 gg((unsigned)nchunks, (unsigned)H);
  const float scale_log2 = (float)(1.0 / std::sqrt((double)d)) * pia::kLog2e;
  const bool bd = bidir != 0;
  const dim3 gt((unsigned)tiles, (unsigned)(B * H));
  const char* why = "backward kernel launch";
  using bf = __nv_bfloat16;
  if (tc) {
    // the forward on the tensor cores for out, lse and D = dO . out (from its fp32 output rows),
    // then the dq pass and the dk/dv pass on the tensor cores.  Split: the forward's skip partials
    // go to dq (rows * (2d + 4) <= rows * 4d bytes, written over by the dq passes after it), and
    // each pass runs over the skips in the residue view first, then over the window (S = 0),
    // adding to what the first wrote.
    const long long off = (bwd_ws_bytes(B, H, n, d, true) - rows * 2LL * d - rows * 4LL);
    bf* out_ws = reinterpret_cast<bf*>(static_cast<char*>(scratch) + off);
    float* lse_ws = reinterpret_cast<float*>(static_cast<char*>(scratch) + off + rows * 2LL * d);
    e = d == 128 ? pia::launch_fwd_tc_with_dot<128>(q, k, v, w_g, b_g, dout, out_ws, lse_ws, rs.D, rs.lse2, rs.bl2,
                                                    rs.bp2, B, H, n, k_win, pi, S, bd, split, dq, s, &why)
                 : pia::launch_fwd_tc_with_dot<64>(q, k, v, w_g, b_g, dout, out_ws, lse_ws, rs.D, rs.lse2, rs.bl2,
                                                   rs.bp2, B, H, n, k_win, pi, S, bd, split, dq, s, &why);
    pia::tcb::BParams bp;
    bp.w_g = w_g;
    bp.b_g = b_g;
    bp.lse = lse_ws;
    bp.Dr = rs.D;
    bp.dq = dq;
    bp.dz = rs.dz;
    bp.part_w = part_w;
    bp.part_b = part_b;
    bp.H = H;
    bp.n = n;
    bp.kwin = k_win;
    bp.pi = pi;
    bp.S = S;
    bp.scale_log2 = scale_log2;
    bp.bidir = bd ? 1 : 0;
    bp.acc = 0;
    pia::tcb::KParams kp;
    kp.lse2 = rs.lse2;
    kp.Dr = rs.D;
    kp.bl2 = rs.bl2;
    kp.bp2 = rs.bp2;
    kp.dk = dk;
    kp.dv = dv;
    kp.n = n;
    kp.kwin = k_win;
    kp.pi = pi;
    kp.S = S;
    kp.scale_log2 = scale_log2;
    kp.bidir = bd ? 1 : 0;
    kp.acc = 0;
    using namespace pia::tcb;
    // The forward wrote every row term the two passes read (lse, D, the log2 priors), so the
    // dk/dv passes run on the side stream beside the dq passes: they read what the forward wrote
    // and write only dk and dv.  The side stream joins back before anything after them on `s`
    // (the gate's final sums wait for the dq passes alone; the scratch release for both).
    SideStream* side = nullptr;
    bool forked = false;
    if (e == cudaSuccess) {
      if ((e = side_stream(&side)) == cudaSuccess && (e = side_fork(*side, s)) == cudaSuccess)
        forked = true;
      else
        why = "backward side stream";
    }
    if (forked) {
      const cudaStream_t s2 = side->stream;
      if (split) {
        e = d == 128 ? launch_bwd_dkv<128, 1>(q, k, v, dout, kp, B * H, s2, &why)
                     : launch_bwd_dkv<64, 1>(q, k, v, dout, kp, B * H, s2, &why);
        kp.S = 0;
        kp.acc = 1;
      }
      if (e == cudaSuccess)
        e = d == 128 ? launch_bwd_dkv<128, 0>(q, k, v, dout, kp, B * H, s2, &why)
                     : launch_bwd_dkv<64, 0>(q, k, v, dout, kp, B * H, s2, &why);
    }
    if (split) {
      if (e == cudaSuccess)
        e = d == 128 ? launch_bwd_dq<128, 1>(q, k, v, dout, bp, B * H, s, &why)
                     : launch_bwd_dq<64, 1>(q, k, v, dout, bp, B * H, s, &why);
      bp.S = 0;  // the window pass
      bp.acc = 1;
    }
    if (e == cudaSuccess)
      e = d == 128 ? launch_bwd_dq<128, 0>(q, k, v, dout, bp, B * H, s, &why)
                   : launch_bwd_dq<64, 0>(q, k, v, dout, bp, B * H, s, &why);
    // the gate's partial sums come from the window dq pass, one per (b, query tile); their final
    // sums run while the side stream may still be busy
    if (e == cudaSuccess) pia::bwd_gate_final_kernel<<<dim3((unsigned)H, (unsigned)((d + 31) / 32)), 1024, 0, s>>>(
          part_w, part_b, dw_g, db_g, (int)nchunks, d);
    if (forked) {  // always, whatever failed above: `s` must not run ahead of the side stream's work
      const cudaError_t ej = side_join(*side, s);
      if (e == cudaSuccess && ej != cudaSuccess) {
        e = ej;
        why = "backward side stream join";
      }
    }
  } else if (dtype == PI_ATTN_F32) {
    e = launch_bwd<float>(q, k, v, w_g, b_g, dout, dq, dk, dv, rs, gt, H, n, d, k_win, pi, S, scale_log2, bd, s);
    if (e == cudaSuccess)
      pia::bwd_gate_partial_kernel<float><<<gg, 256, 0, s>>>((const float*)q, rs.dz, part_w, part_b, B, H, n, d);
  } else {
    e = launch_bwd<bf>(q, k, v, w_g, b_g, dout, dq, dk, dv, rs, gt, H, n, d, k_win, pi, S, scale_log2, bd, s);
    if (e == cudaSuccess)
      pia::bwd_gate_partial_kernel<bf><<<gg, 256, 0, s>>>((const bf*)q, rs.dz, part_w, part_b, B, H, n, d);
  }
  if (e == cudaSuccess && !tc) pia::bwd_gate_final_kernel<<<dim3((unsigned)H, (unsigned)((d + 31) / 32)), 1024, 0, s>>>(
        part_w, part_b, dw_g, db_g, (int)nchunks, d);
  if (e == cudaSuccess) e = cudaGetLastError();
  cudaError_t e2 = workspace ? cudaSuccess : cudaFreeAsync(scratch, s);
  if (e != cudaSuccess) return cuda_fail(e, why);
  if (e2 != cudaSuccess) return cuda_fail(e2, "backward scratch release");
  return ok();
}

long long pi_attn_bwd_host_workspace_bytes(int B, int H, int n, int d, pi_attn_dtype dtype, pi_attn_bwd_path path,
                                           int chunk_heads) {
  if (B < 1 || H < 1 || n < 1 || d < 1 || chunk_heads < 0 || (dtype != PI_ATTN_F32 && dtype != PI_ATTN_BF16) ||
      path < PI_ATTN_BWD_AUTO || path > PI_ATTN_BWD_TC_SPLIT)
    return -1;
  const int hc = host_chunk_heads(H, chunk_heads);
  const long long per = (long long)B * hc * n * d;
  const long long set = 4 * round256(per * (long long)elem_size(dtype)) + 3 * round256(per * 4);
  return kHostSets * set + round256(pi_attn_bwd_workspace_bytes_ex(B, hc, n, d, dtype, path));
}

pi_attn_status pi_attn_bwd_host(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                                const void* dout, float* dq, float* dk, float* dv, float* dw_g, float* db_g, int B,
                                int H, int n, int d, int k_win, int pi, int S, pi_attn_dtype dtype, int bidir,
                                pi_attn_bwd_path path, int chunk_heads, void* workspace, long long workspace_bytes,
                                void* stream) {
  if (!q || !k || !v || !dout || !dq || !dk || !dv) return fail(PI_ATTN_EINVAL, "null host tensor pointer");
  if (!w_g || !b_g || !dw_g || !db_g) return fail(PI_ATTN_EINVAL, "null gate parameter or gradient pointer");
  if (chunk_heads < 0) return fail(PI_ATTN_EINVAL, "chunk_heads must be >= 0 (got %d)", chunk_heads);
  static const char dummy[16] __attribute__((aligned(16))) = {0};
  pi_attn_status st = check_common(dummy, dummy, dummy, w_g, b_g, dummy, B, H, n, d, k_win, pi, S, dtype);
  if (st != PI_ATTN_OK) return st;
  const int hc = host_chunk_heads(H, chunk_heads);
  bool tc = false, split = false;  // (each chunk is a [B, chunk_heads, n, d] problem)
  if ((st = bwd_route(B, hc, n, d, k_win, pi, S, dtype, bidir, path, &tc, &split)) != PI_ATTN_OK) return st;
  const long long need = pi_attn_bwd_host_workspace_bytes(B, H, n, d, dtype, path, chunk_heads);
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
    return fail(PI_ATTN_EINVAL, "workspace must be a 256-byte aligned device pointer");
  if (workspace_bytes < need)
    return fail(PI_ATTN_EINVAL, "workspace of %lld bytes, the call needs %lld", workspace_bytes, need);
  const size_t elem = elem_size(dtype);
  const long long per = (long long)B * hc * n * d;
  const long long ti = round256(per * (long long)elem), to = round256(per * 4), set_bytes = 4 * ti + 3 * to;
  char* const ws = static_cast<char*>(workspace);
  void* const bwd_ws = ws + kHostSets * set_bytes;
  const long long bwd_ws_bytes_chunk = round256(pi_attn_bwd_workspace_bytes_ex(B, hc, n, d, dtype, path));
  cudaStream_t s = as_stream(stream);

  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe* hp = nullptr;
  cudaError_t e = host_pipe(&hp);
  if (e != cudaSuccess) return cuda_fail(e, "copy streams");
  if ((e = cudaEventRecord(hp->start, s)) != cudaSuccess || (e = cudaStreamWaitEvent(hp->in, hp->start, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(hp->out, hp->start, 0)) != cudaSuccess)
    return cuda_fail(e, "copy streams");
  // a chunk holds heads [h0, h0 + h) of every b: in host memory B slabs of h heads, H heads apart
  const size_t head_in = (size_t)n * d * elem, head_out = (size_t)n * d * 4;
  int c = 0;
  for (int h0 = 0; h0 < H && st == PI_ATTN_OK && e == cudaSuccess; h0 += hc, ++c) {
    const int h = hc < H - h0 ? hc : H - h0, set = c % kHostSets;
    char* const base = ws + set * set_bytes;
    void* din[4] = {base, base + ti, base + 2 * ti, base + 3 * ti};  // q, k, v, dout
    float* dgr[3] = {reinterpret_cast<float*>(base + 4 * ti), reinterpret_cast<float*>(base + 4 * ti + to),
                     reinterpret_cast<float*>(base + 4 * ti + 2 * to)};  // dq, dk, dv
    const void* hin[4] = {q, k, v, dout};
    float* hgr[3] = {dq, dk, dv};
    if (c >= kHostSets && (e = cudaStreamWaitEvent(hp->in, hp->freed[set], 0)) != cudaSuccess) break;
    for (int x = 0; x < 4 && e == cudaSuccess; ++x)
      e = cudaMemcpy2DAsync(din[x], h * head_in, static_cast<const char*>(hin[x]) + h0 * head_in, (size_t)H * head_in,
                            h * head_in, B, cudaMemcpyHostToDevice, hp->in);
    if (e != cudaSuccess || (e = cudaEventRecord(hp->loaded[set], hp->in)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(s, hp->loaded[set], 0)) != cudaSuccess)
      break;
    // the chunk as a [B, h, n, d] problem: its heads' gate parameters, and their gradients (every b
    // is in the chunk, so the gate gradients of these heads are complete) straight into dw_g, db_g
    st = pi_attn_bwd_ex(din[0], din[1], din[2], w_g + (long long)h0 * d, b_g + h0, din[3], dgr[0], dgr[1], dgr[2],
                        dw_g + (long long)h0 * d, db_g + h0, B, h, n, d, k_win, pi, S, dtype, bidir, path, bwd_ws,
                        bwd_ws_bytes_chunk, stream);
    if (st != PI_ATTN_OK) break;
    if ((e = cudaEventRecord(hp->computed[set], s)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(hp->out, hp->computed[set], 0)) != cudaSuccess)
      break;
    for (int x = 0; x < 3 && e == cudaSuccess; ++x)
      e = cudaMemcpy2DAsync(reinterpret_cast<char*>(hgr[x]) + h0 * head_out, (size_t)H * head_out, dgr[x],
                            h * head_out, h * head_out, B, cudaMemcpyDeviceToHost, hp->out);
    if (e != cudaSuccess || (e = cudaEventRecord(hp->freed[set], hp->out)) != cudaSuccess) break;
  }
  cudaError_t ej = cudaEventRecord(hp->join_in, hp->in);
  if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, hp->join_in, 0);
  if (ej == cudaSuccess) ej = cudaEventRecord(hp->join_out, hp->out);
  if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, hp->join_out, 0);
  if (st != PI_ATTN_OK) return st;
  if (e != cudaSuccess) return cuda_fail(e, "host-buffer chunk copies");
  if (ej != cudaSuccess) return cuda_fail(ej, "joining the copy streams");
  return ok();
}

pi_attn_status pi_attn_bwd(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                           const void* dout, float* dq, float* dk, float* dv, float* dw_g, float* db_g, int B, int H,
                           int n, int d, int k_win, int pi, int S, pi_attn_dtype dtype, int bidir, void* workspace,
                           long long workspace_bytes, void* stream) {
  return pi_attn_bwd_ex(q, k, v, w_g, b_g, dout, dq, dk, dv, dw_g, db_g, B, H, n, d, k_win, pi, S, dtype, bidir,
                        PI_ATTN_BWD_SIMT, workspace, workspace_bytes, stream);
}

pi_attn_status pi_attn_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned word = 0;
  e = cudaMemcpyFromSymbol(&word, pia::g_error_word, sizeof word);
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (word) {
    const unsigned zero = 0;
    cudaMemcpyToSymbol(pia::g_error_word, &zero, sizeof zero);
    return fail(PI_ATTN_EDEVICE, "device error flags 0x%x:%s%s%s", word,
                (word & pia::kErrWaitTimeout) ? " pipeline-wait-timeout" : "",
                (word & pia::kErrCacheLen) ? " cache_len-out-of-range" : "",
                (word & pia::kErrInternal) ? " internal-check" : "");
  }
  return ok();
}

}  // extern "C"
