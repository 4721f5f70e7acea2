/*
 * pi_attn.h -- C ABI of the pi-attention forward operator for NVIDIA B200 (sm_100a).
 *
 * The operator ("pi-Attention: Periodic Sparse Transformers for Efficient Long-Context Modeling",
 * gist.science summary, section 2 "Methodology", Core Components): every query row i of every
 * (batch b, head h) attends, under ONE softmax, to the union of
 *   - its causal ring-local window  L(i) = { j : max(0, i - k) <= j <= i }  (itself + k before),
 *   - its periodic backward skips   P(i) = { i - m*pi : 1 <= m <= S, m*pi > k, i - m*pi >= 0 }
 *     (a skip that lands inside the window is dropped, so every key is counted once),
 * with a per-token, per-head gate alpha = sigmoid(q_i . w_g[h] + b_g[h]) on the unscaled query,
 * added as a log-prior: log(alpha) on window logits, log(1 - alpha) on skip logits, before the
 * softmax (section "Dynamic Adaptive Fusion").  Logits are scaled by tau = 1/sqrt(d); the prior
 * is not scaled.  Outputs:
 *   out_i = sum_j softmax_j(s) v_j          lse_i = ln sum_j exp(s_j)   (natural log)
 *
 * Conventions shared by every entry point
 *   - Tensors are contiguous, row-major, innermost dimension d.  q/k/v/out of prefill are
 *     [B, H, n, d]; decode q/out are [B, H, d] and the caches [B, H, n_cache, d]; lse is [B, H, n]
 *     (prefill) or [B, H] (decode), fp32.  w_g is [H, d] fp32, b_g is [H] fp32.
 *   - dtype names the storage type of q, k, v, caches and out: PI_ATTN_F32 (fp32) or PI_ATTN_BF16
 *     (bfloat16).  Arithmetic is fp32 (bf16 products on tensor cores accumulate in fp32); out is
 *     rounded once, to nearest even, into dtype.
 *   - All pointers are DEVICE pointers owned by the caller (pi_attn_fwd_host and pi_attn_bwd_host
 *     take host buffers instead); the library keeps no reference after the call returns and holds no memory
 *     allocation of its own between calls, with two exceptions stated at their entry points: the
 *     fixed device array of the decode for callers that cannot allocate, and the streams and
 *     events it creates once per device, on first use, for the tensor-core backward and the
 *     host-buffer entry points (kept until the process exits).  Tensor pointers must be 16-byte aligned
 *     and d * sizeof(dtype) a multiple of 16 bytes.
 *   - `stream` is a cudaStream_t (NULL: the legacy default stream).  Calls only enqueue work: they
 *     are asynchronous and stream-ordered.  Argument errors are returned synchronously and then
 *     nothing is enqueued.  Errors that only a kernel can see (a cache length out of range, an
 *     internal wait that gave up) set a device-side error word that pi_attn_check() reads.
 *   - Entry points are thread-safe; the device error word is shared by all streams of a device.
 */
#ifndef PI_ATTN_H
#define PI_ATTN_H

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PI_ATTN_OK = 0,
    PI_ATTN_EINVAL = 1,        /* invalid argument: null pointer, size out of range, misalignment */
    PI_ATTN_EUNSUPPORTED = 2,  /* valid request the library does not implement (e.g. head size) */
    PI_ATTN_ECUDA = 3,         /* a CUDA runtime call or kernel launch failed */
    PI_ATTN_EDEVICE = 4        /* a kernel reported an error through the device error word */
} pi_attn_status;

typedef enum { PI_ATTN_F32 = 0, PI_ATTN_BF16 = 1 } pi_attn_dtype;

/* Kernel choice for pi_attn_fwd_ex. */
typedef enum {
    PI_ATTN_PATH_AUTO = 0,      /* tensor-core kernel where it applies (bf16, d in {64, 128}, B*H <= 65535),
                                   else SIMT */
    PI_ATTN_PATH_SIMT = 1,      /* CUDA-core kernel: every dtype, d <= 256 */
    PI_ATTN_PATH_TC = 2,        /* tcgen05/TMEM kernels only (single pass or split, chosen by shape);
                                   PI_ATTN_EUNSUPPORTED where they do not apply */
    PI_ATTN_PATH_TC_FUSED = 3,  /* tensor cores, window and skips in one pass */
    PI_ATTN_PATH_TC_SPLIT = 4   /* tensor cores, skips in a residue-class pass over the whole periods,
                                   rows [0, (n / pi) pi) (scratch of B*H*n*(2d + 4) bytes from
                                   cudaMallocAsync on `stream`), then the window pass merging them;
                                   query tiles reaching past the whole periods take the single pass.
                                   Causal; needs n >= pi and a skip outside the window */
} pi_attn_path;

/* Prefill forward.  Cited passage: the Core Components (window, skips, gate as log-prior, one
 * softmax over the union) and "Execution & Scheduling" (local sweep on tensor cores, periodic
 * strided gather, fusion) of the pi-Attention method section.
 *   q, k, v   [B, H, n, d] in dtype                        (read)
 *   w_g [H, d], b_g [H]  fp32 gate parameters               (read)
 *   out       [B, H, n, d] in dtype                         (written)
 *   lse       [B, H, n] fp32, natural log; may be NULL     (written)
 *   B, H, n >= 1; d: multiple of 4 (fp32) or 8 (bf16), 1..256; k_win >= 0; pi >= 1; S >= 0.
 * Returns PI_ATTN_OK once the work is enqueued. */
pi_attn_status pi_attn_fwd(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                           void* out, float* lse, int B, int H, int n, int d, int k_win, int pi, int S,
                           pi_attn_dtype dtype, void* stream);

/* pi_attn_fwd with an explicit kernel choice (see pi_attn_path).  Same arguments and results. */
pi_attn_status pi_attn_fwd_ex(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                              void* out, float* lse, int B, int H, int n, int d, int k_win, int pi, int S,
                              pi_attn_dtype dtype, pi_attn_path path, void* stream);

/* pi_attn_fwd_ex with a caller-provided device workspace for the split path's skip partials, so
 * that the call allocates nothing (and can be captured in a CUDA graph without memory nodes).
 *   workspace        device pointer, 16-byte aligned, owned by the caller; NULL = allocate as
 *                    pi_attn_fwd_ex does (cudaMallocAsync on `stream`, freed stream-ordered)
 *   workspace_bytes  its size; at least the scratch_bytes pi_attn_fwd_plan reports for the same
 *                    arguments (0 when the call runs a single pass), else PI_ATTN_EINVAL
 * The workspace is read and written by the call's kernels only: it may be reused by the next call
 * on the same stream, and must not be touched by other streams while the call runs. */
pi_attn_status pi_attn_fwd_ws(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                              void* out, float* lse, int B, int H, int n, int d, int k_win, int pi, int S,
                              pi_attn_dtype dtype, pi_attn_path path, void* workspace, long long workspace_bytes,
                              void* stream);

/* One shard of a causal prefill, for a sequence split by rows across devices.  Cited passages: the
 * gist.science summaries of "pi-Attention: Periodic Sparse Transformers for Efficient Long-Context
 * Modeling" -- Dutch, sections 2 and 3 (the fixed strides give a communication pattern known in
 * advance, suited to NCCL/NVLink), English, Hardware Efficiency (less inter-device traffic than
 * random sparse patterns).  A shard owning sequence rows [row0, row0 + n_q) reads keys back to
 * row0 - max(k_win, S*pi) (skips only where m*pi > k_win), so it needs that halo of K/V rows from
 * the shards before it and nothing from the shards after it.
 *   q, out  [B, H, n_q, d]   sequence rows row0 .. row0 + n_q - 1 (lse [B, H, n_q], may be NULL)
 *   k, v    [B, H, n_kv, d]  sequence rows kv0 .. kv0 + n_kv - 1: the halo, then the shard's rows
 * Where row0 and kv0 are whole periods (multiples of pi) and a sequence of n_q rows would take the
 * split path, the shard takes it too (the residue-class pass over its whole periods, with its
 * scratch of B*H*n_q*(2d + 4) bytes from cudaMallocAsync on `stream`, then the window pass);
 * otherwise the single tensor-core pass, which allocates nothing.  Either way every row is computed
 * by the same kernels as the whole sequence's call on that path; the single pass gives it the same
 * bits, the split path up to the rounding of the tiles it groups the row with.
 * PI_ATTN_EINVAL unless kv0 <= max(0, row0 - max(k_win, S*pi)) (the halo reaches every key read)
 * and kv0 + n_kv >= row0 + n_q (the k/v rows reach the shard's last row), plus the checks of
 * pi_attn_fwd; bf16 with d in {64, 128}, else PI_ATTN_EUNSUPPORTED.  All pointers are device
 * pointers owned by the caller. */
pi_attn_status pi_attn_fwd_shard(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                                 void* out, float* lse, int B, int H, int n_q, int n_kv, long long row0,
                                 long long kv0, int d, int k_win, int pi, int S, pi_attn_dtype dtype, void* stream);

/* pi_attn_fwd_shard with a caller-provided device workspace for the split path's skip partials
 * (16-byte aligned, owned by the caller; at least pi_attn_fwd_shard_scratch_bytes bytes; NULL =
 * allocate as pi_attn_fwd_shard does), so that the call allocates nothing.  Errors as
 * pi_attn_fwd_shard, plus PI_ATTN_EINVAL for a misaligned or too small workspace. */
pi_attn_status pi_attn_fwd_shard_ws(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                                    void* out, float* lse, int B, int H, int n_q, int n_kv, long long row0,
                                    long long kv0, int d, int k_win, int pi, int S, pi_attn_dtype dtype,
                                    void* workspace, long long workspace_bytes, void* stream);
/* Scratch bytes a shard call with these arguments takes: B*H*n_q*(2d + 4) where it runs the split
 * path, 0 where it runs the single pass; -1 for invalid sizes. */
long long pi_attn_fwd_shard_scratch_bytes(int B, int H, int n_q, long long row0, long long kv0, int d, int k_win,
                                          int pi, int S);

/* Bidirectional prefill forward (the non-causal variant).  Cited passage: the Core Components of
 * the pi-Attention method section -- the local neighbourhood reaches both forward and backward,
 * and in bidirectional settings the skips also reach i + pi.  Row i of a sequence of n tokens
 * attends, under one softmax, to
 *   L(i) = { j : max(0, i - k_win) <= j <= min(n - 1, i + k_win) }        prior log(alpha)
 *   P(i) = { i - m*pi, i + m*pi : 1 <= m <= S, m*pi > k_win, 0 <= key < n } prior log(1 - alpha)
 * Same arguments, layouts, ownership and errors as pi_attn_fwd_ex.  PI_ATTN_PATH_TC_SPLIT (and the
 * automatic choice of it for long contexts) needs n % pi == 0 and a skip outside the window, else
 * PI_ATTN_EUNSUPPORTED: its residue-class pass takes both skip bands of a class, and its scratch
 * comes from cudaMallocAsync on `stream` as for pi_attn_fwd_ex; the other paths allocate nothing. */
pi_attn_status pi_attn_fwd_bidir(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                                 void* out, float* lse, int B, int H, int n, int d, int k_win, int pi, int S,
                                 pi_attn_dtype dtype, pi_attn_path path, void* stream);

/* pi_attn_fwd_ex over inputs and outputs in HOST memory, as a pipeline of chunks.  Cited
 * passage: "Execution & Scheduling" (the operator streams a long context through the device).
 * The (b, h) heads are taken chunk_heads at a time (within one b; 0 = about a thirty-second of H): the
 * copy of the next chunk's q, k and v to the device, the computation of this chunk (the same
 * kernels and bits as pi_attn_fwd_ex on device copies of the same inputs) and the copy of the
 * previous chunk's out and lse back overlap, on two copy streams the library creates once per
 * device and on `stream` for the computation.
 *   q, k, v   HOST [B, H, n, d] in dtype, read only; page-locked (cudaHostAlloc or pinned) for the
 *             copies to overlap -- pageable memory works, but each copy then blocks the host
 *   out       HOST [B, H, n, d] in dtype; lse HOST fp32 [B, H, n] or NULL
 *   w_g, b_g  DEVICE, as for pi_attn_fwd (the gate parameters stay resident)
 *   workspace DEVICE, 256-byte aligned, pi_attn_fwd_host_workspace_bytes(B, H, n, d, dtype,
 *             chunk_heads) bytes, owned by the caller (three rotating chunk buffers and the split
 *             path's scratch)
 * Ordering: the copies start after the work already enqueued on `stream`, and `stream` waits for
 * all of the call's copies before anything enqueued on it after the call; out and lse are
 * complete on the host once `stream` has been synchronized.  The host buffers must stay valid
 * and untouched until then.  Errors as pi_attn_fwd_ex, plus PI_ATTN_EINVAL for a NULL host
 * pointer, a negative chunk_heads or a workspace that is missing, misaligned or too small.
 * Causal rule only; not for graph capture with pageable host memory. */
pi_attn_status pi_attn_fwd_host(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                                void* out, float* lse, int B, int H, int n, int d, int k_win, int pi, int S,
                                pi_attn_dtype dtype, pi_attn_path path, int chunk_heads, void* workspace,
                                long long workspace_bytes, void* stream);
/* Device workspace bytes pi_attn_fwd_host needs for these sizes; -1 for invalid sizes. */
long long pi_attn_fwd_host_workspace_bytes(int B, int H, int n, int d, pi_attn_dtype dtype, int chunk_heads);

/* What a pi_attn_fwd_ex call with these arguments would launch, without launching anything:
 * *launches = number of kernel launches (1 for a single pass; 2 or 3 for the split: the residue pass,
 * then the band-merge pass and / or the single pass over the tiles past the whole periods),
 * *scratch_bytes =
 * device scratch it needs (0 for a single pass): taken from cudaMallocAsync on the stream, or the
 * workspace given to pi_attn_fwd_ws.  Returns
 * PI_ATTN_EUNSUPPORTED / PI_ATTN_EINVAL exactly where pi_attn_fwd_ex would. */
pi_attn_status pi_attn_fwd_plan(int B, int H, int n, int d, int k_win, int pi, int S, pi_attn_dtype dtype,
                                pi_attn_path path, int* launches, long long* scratch_bytes);

/* Single-step decode.  Cited passage: "Inference" under "Execution & Scheduling" of the
 * pi-Attention method section (a new token reads its window and its periodic skips).  For each
 * (b, h) the query q[b, h] is the token at position len_b - 1 of a cache that already holds it,
 * with len_b = cache_len[b] (or n_cache when cache_len is NULL); it attends to cache rows by the
 * prefill rule.  Cache rows outside the window and skips are never read.
 *   q        [B, H, d] dtype                  kcache, vcache [B, H, n_cache, d] dtype
 *   w_g, b_g as for prefill                   cache_len: device int32 [B] or NULL
 *   out      [B, H, d] dtype                  lse: [B, H] fp32 or NULL
 * A cache_len entry outside [1, n_cache] sets the device error word (read by pi_attn_check) and
 * that sequence's out/lse are written as NaN. */
pi_attn_status pi_attn_decode(const void* q, const void* kcache, const void* vcache, const float* w_g,
                              const float* b_g, const int* cache_len, void* out, float* lse, int B, int H,
                              int n_cache, int d, int k_win, int pi, int S, pi_attn_dtype dtype, void* stream);

/* pi_attn_decode for callers that cannot allocate device memory.  (The pages describe no such
 * call: this is a property of the library, not of the method.)
 *
 * pi_attn_decode takes a small workspace from cudaMallocAsync on `stream` whenever it spreads one
 * (b, h) over several CTAs, which it does when B*H is too small to fill the GPU.  Some callers
 * cannot let a library allocate.  For example, a process whose device memory is reserved up front
 * by its own allocator has no room, or no quota, for a library allocation.  A runtime with a fixed
 * memory plan must know every byte in advance.  Such callers use this entry point: same
 * arguments, same results, no allocation and no free.  The caller still passes every input and
 * output.  The workspace is a fixed device array inside the library of 4 MiB (1,048,576 floats),
 * which every GPU that loads the library holds until the process exits.
 *   - Sizes: bf16 with d in {64, 128}.  A call whose split needs more than the 4 MiB
 *     (B*H * splits * (d + 2) floats) returns PI_ATTN_EINVAL and enqueues nothing; with the
 *     library's split rule this needs a B*H far above what splits at all.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress), with
 *     that device current.  Make that first call before any stream capture.
 *   - Every call shares the one array, and it keeps the last call's contents; the kernels
 *     overwrite every slot they read, so nothing needs clearing.  Two calls whose kernels overlap
 *     on the GPU (different streams, no ordering between them) race on the array: order them on
 *     one stream or with events.
 *   - Errors as for pi_attn_decode. */
pi_attn_status pi_attn_decode_noalloc(const void* q, const void* kcache, const void* vcache, const float* w_g,
                                      const float* b_g, const int* cache_len, void* out, float* lse, int B, int H,
                                      int n_cache, int d, int k_win, int pi, int S, pi_attn_dtype dtype,
                                      void* stream);

/* Backward: the gradients of a scalar loss through out, given dout = dLoss/dout.  Not printed on
 * the pages; it is the chain rule through the forward (prefill, causal or, with bidir = 1, the
 * bidirectional rule) that the pages' training results rely on.  With p_ij the softmax weights:
 *   D_i = dout_i . out_i,  ds_ij = p_ij (dout_i . v_j - D_i)
 *   dq_i = tau sum_j ds_ij k_j + dz_i w_g[h],  dk_j = tau sum_i ds_ij q_i,  dv_j = sum_i p_ij dout_i
 *   dz_i = (1 - alpha_i) sum_{j in L(i)} ds_ij - alpha_i sum_{j in P(i)} ds_ij
 *   dw_g[h] = sum_{b,i} dz_i q_i,  db_g[h] = sum_{b,i} dz_i
 *   q, k, v, dout   [B, H, n, d] in dtype (read); w_g [H, d], b_g [H] fp32 (read)
 *   dq, dk, dv      [B, H, n, d] fp32 (written whole, 16-byte aligned)
 *   dw_g [H, d], db_g [H] fp32 (written whole)
 *   workspace       device scratch of pi_attn_bwd_workspace_bytes(B, H, n, d) bytes, 16-byte aligned,
 *                   or NULL (then taken from cudaMallocAsync on the stream and released after)
 * The forward is recomputed from the inputs; nothing of a forward call is needed.  Results do not
 * depend on scheduling (no atomics).  Same argument rules and errors as pi_attn_fwd. */
long long pi_attn_bwd_workspace_bytes(int B, int H, int n, int d);
pi_attn_status pi_attn_bwd(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                           const void* dout, float* dq, float* dk, float* dv, float* dw_g, float* db_g, int B, int H,
                           int n, int d, int k_win, int pi, int S, pi_attn_dtype dtype, int bidir, void* workspace,
                           long long workspace_bytes, void* stream);

/* The backward with a choice of kernels.  PI_ATTN_BWD_SIMT is pi_attn_bwd: the forward recomputed
 * in fp32 on CUDA cores with every product in fp32.  The tensor-core paths run the forward on the
 * tensor cores for lse and D_i = dout_i . out_i (from its fp32 output rows), then a dq pass and a
 * dk/dv pass on the tensor cores (S, dP and their transposes by tcgen05 in fp32; P and ds rounded
 * to bf16 for dQ += dS K, dV += P^T dO, dK += dS^T Q); their gradients carry those bf16 roundings
 * (relative errors of order 2^-9), against fp32 arithmetic for the SIMT path.  bf16 with d in
 * {64, 128} (else PI_ATTN_EUNSUPPORTED).
 *   PI_ATTN_BWD_TC_FUSED  each pass walks the window and the skips of a row (or key) in one sweep.
 *   PI_ATTN_BWD_TC_SPLIT  the forward's split reading for long contexts: the forward, the dq pass
 *                         and the dk/dv pass each run once over the skips alone in the residue-class
 *                         view (the skip keys of a row form a dense band there) and once over the
 *                         window alone; the skip passes use dq as scratch before writing it.  The
 *                         causal rule with n % pi == 0 (the backward's residue view holds every
 *                         row) and a skip outside the window, else PI_ATTN_EUNSUPPORTED.
 *   PI_ATTN_BWD_TC        tensor cores, fused or split chosen by shape as for PI_ATTN_PATH_TC.
 *   PI_ATTN_BWD_AUTO      PI_ATTN_BWD_TC where the tensor cores apply, else SIMT.
 * The workspace is pi_attn_bwd_workspace_bytes_ex(B, H, n, d, dtype, path) bytes (the tensor-core
 * paths add the forward's out and lse); other arguments and errors as pi_attn_bwd.
 * Streams (tensor-core paths): the dk/dv pass runs on a second stream that the library creates
 * once per device, forked from `stream` after the forward and joined back into it before the call
 * returns, so all work of the call is ordered before whatever the caller enqueues on `stream`
 * next; a graph capture of `stream` captures both branches.  The first tensor-core backward on a
 * device creates that stream and two events, so make it before any graph capture. */
typedef enum {
    PI_ATTN_BWD_AUTO = 0,
    PI_ATTN_BWD_SIMT = 1,
    PI_ATTN_BWD_TC = 2,
    PI_ATTN_BWD_TC_FUSED = 3,
    PI_ATTN_BWD_TC_SPLIT = 4
} pi_attn_bwd_path;
long long pi_attn_bwd_workspace_bytes_ex(int B, int H, int n, int d, pi_attn_dtype dtype, pi_attn_bwd_path path);
pi_attn_status pi_attn_bwd_ex(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                              const void* dout, float* dq, float* dk, float* dv, float* dw_g, float* db_g, int B,
                              int H, int n, int d, int k_win, int pi, int S, pi_attn_dtype dtype, int bidir,
                              pi_attn_bwd_path path, void* workspace, long long workspace_bytes, void* stream);

/* pi_attn_bwd_ex over inputs and gradients in HOST memory, as a pipeline of chunks of heads (as
 * pi_attn_fwd_host does for the prefill).  A chunk is chunk_heads heads of every b (0 = about a
 * thirty-second of H), so the gate gradients of its heads are complete within it; its q, k, v and
 * dout are copied in, its gradients computed by pi_attn_bwd_ex on `stream` (the same kernels and
 * bits as a pi_attn_bwd_ex call on device copies of the same inputs) and dq, dk, dv copied out,
 * the copies of neighbouring chunks overlapping each chunk's kernels on the library's two copy
 * streams.
 *   q, k, v, dout  HOST [B, H, n, d] in dtype, read only (page-locked for the copies to overlap)
 *   dq, dk, dv     HOST fp32 [B, H, n, d]
 *   w_g, b_g       DEVICE, as for pi_attn_bwd; dw_g, db_g DEVICE fp32 [H, d] and [H]
 *   workspace      DEVICE, 256-byte aligned, pi_attn_bwd_host_workspace_bytes(B, H, n, d, dtype,
 *                  path, chunk_heads) bytes, owned by the caller
 * Ordering as for pi_attn_fwd_host: the gradients are on the host once `stream` has been
 * synchronized.  Errors as pi_attn_bwd_ex, plus PI_ATTN_EINVAL for a NULL host pointer, a negative
 * chunk_heads or a workspace that is missing, misaligned or too small. */
pi_attn_status pi_attn_bwd_host(const void* q, const void* k, const void* v, const float* w_g, const float* b_g,
                                const void* dout, float* dq, float* dk, float* dv, float* dw_g, float* db_g, int B,
                                int H, int n, int d, int k_win, int pi, int S, pi_attn_dtype dtype, int bidir,
                                pi_attn_bwd_path path, int chunk_heads, void* workspace, long long workspace_bytes,
                                void* stream);
/* Device workspace bytes pi_attn_bwd_host needs; -1 for invalid arguments. */
long long pi_attn_bwd_host_workspace_bytes(int B, int H, int n, int d, pi_attn_dtype dtype, pi_attn_bwd_path path,
                                           int chunk_heads);

/* Decode over a compact ring cache (constant memory per sequence, constant-time update).  Cited
 * passage: "Execution & Scheduling" -- caches updated in constant time at inference.  Position j of
 * sequence b lives in slot j mod capacity of kcache / vcache [B, H, capacity, d]; the query is the
 * token at position cache_len[b] - 1 (any value >= 1, also beyond capacity) and reads L and P as in
 * pi_attn_decode.  capacity must be >= max(k_win, S*pi) + 1, the farthest a step can still reach
 * (PI_ATTN_EINVAL otherwise); cache_len is required.  bf16 with d in {64, 128}
 * (PI_ATTN_EUNSUPPORTED otherwise).  Other arguments, errors and the device check of cache_len
 * (>= 1) as for pi_attn_decode. */
pi_attn_status pi_attn_decode_ring(const void* q, const void* kcache, const void* vcache, const float* w_g,
                                   const float* b_g, const int* cache_len, void* out, float* lse, int B, int H,
                                   int capacity, int d, int k_win, int pi, int S, pi_attn_dtype dtype, void* stream);

/* One decode step's new token into the cache, then cache_len[b] += 1 for every b (stream-ordered):
 * row cache_len[b] of every (b, h) -- slot cache_len[b] mod capacity when ring != 0 -- takes
 * k_new / v_new [B, H, d].  kcache, vcache [B, H, capacity, d] and k_new, v_new in dtype, 16-byte
 * aligned; cache_len device int32 [B].  A plain cache (ring = 0) that is full, or a negative
 * cache_len, is reported through the device error word (pi_attn_check) and that b is left as is. */
pi_attn_status pi_attn_cache_append(void* kcache, void* vcache, const void* k_new, const void* v_new, int* cache_len,
                                    int B, int H, int capacity, int d, pi_attn_dtype dtype, int ring, void* stream);

/* Index sets as the kernels see them, for exact comparison.  For query rows i = 0..n-1:
 *   counts [n, 2] int32: |L(i)|, |P(i)|
 *   idx    [n, width] int32: L(i) ascending, then P(i) in order of increasing m, then -1.
 * width must be >= k_win + 1 + S.  Both are device pointers. */
pi_attn_status pi_attn_debug_index_sets(int n, int k_win, int pi, int S, int* counts, int* idx, int width,
                                        void* stream);

/* pi_attn_debug_index_sets for the bidirectional rule (see pi_attn_fwd_bidir): L(i) ascending, then
 * P(i) by increasing m with i - m*pi before i + m*pi.  width must be >= 2*k_win + 1 + 2*S. */
pi_attn_status pi_attn_debug_index_sets_bidir(int n, int k_win, int pi, int S, int* counts, int* idx, int width,
                                              void* stream);

/* Synchronises `stream`, then reads and clears the device error word of the current device.
 * Returns PI_ATTN_EDEVICE if any kernel set it since the last check (pi_attn_last_error() then
 * describes the flags), PI_ATTN_ECUDA if the stream reports a CUDA error, else PI_ATTN_OK. */
pi_attn_status pi_attn_check(void* stream);

/* Static string naming a status code. */
const char* pi_attn_status_string(pi_attn_status status);

/* Description of the last error returned on the calling thread (static storage per thread; ""
 * after a success). */
const char* pi_attn_last_error(void);

/* Library version as major*10000 + minor*100 + patch. */
int pi_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PI_ATTN_H */
