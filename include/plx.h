/*
 * plx.h -- C ABI of libplx: Parallax attention on NVIDIA B200 (sm_100a).
 *
 * Parallax (page 1 "Parallax: Parameterized Local Linear Attention Gives
 * Transformers a 'Second Eye'", opening formula and section 1.3; page 3
 * "Parallax keeps softmax, adds covariance correction branch") is softmax
 * attention with an additive covariance correction.  For query row i,
 *
 *     out_i = o_SA,i - Sigma_KV^(i)^T rho_i
 *
 *     a_ij         = softmax_j(softmax_scale * q_i . k_j)       (page 1, 1.1)
 *     o_SA,i       = sum_j a_ij v_j
 *     mu_i         = sum_j a_ij k_j
 *     Sigma_KV^(i) = sum_j a_ij (k_j - mu_i)(v_j - o_SA,i)^T  (d x d, the
 *                    softmax-weighted covariance of K and V, page 1, 1.3)
 *     rho_i        = the probe (W_R x_i in a model; an input here), contracted
 *                    with the key index of Sigma_KV.
 *
 * rho = 0 gives plain softmax attention (page 3: W_R = 0 recovers softmax).
 * The kernels use the equal one-pass form out = (1 + tbar) o - u with
 * t_j = rho . k_j, tbar = sum a t, u = sum a t v, so a single pass over K and V
 * feeds both branches (page 3: the KV stream is reused by both branches).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers, owned by the caller, contiguous,
 *     row-major in the layouts given below, and 16-byte aligned.  The library
 *     never allocates or frees, and only the diagnostic plx_device_error
 *     synchronises; every other call only enqueues work.
 *   - dtype applies to q, rho, k, v and out alike, unless an entry point takes
 *     an out_dtype or writes fp32 states.  Accumulation is fp32.
 *     PLX_BF16 runs on the tensor cores (prefill) or streams a bf16 cache
 *     (decode); PLX_F32 computes every product in fp32 on the CUDA cores.
 *   - d (head dimension, d_k = d_v) must be 64 or 128; H_q must be a multiple
 *     of H_kv.  Query head h reads key/value head h / (H_q / H_kv).
 *   - stream is a cudaStream_t (NULL = the legacy default stream).  Work runs
 *     asynchronously on it, in order with the caller's other work there.
 *   - Arguments are checked on the host before anything is enqueued; a bad
 *     argument returns PLX_ERR_INVALID_ARGUMENT or PLX_ERR_UNSUPPORTED and
 *     enqueues nothing.  A failed launch returns PLX_ERR_CUDA
 *     (plx_last_cuda_error() gives the cudaError_t).  Faults during execution
 *     surface at the caller's next synchronisation; kernels never wait forever:
 *     a wait that runs out of time records a code readable by
 *     plx_device_error() and the kernel returns.
 *   - Thread safety: calls may come from several host threads; the
 *     per-thread error code is thread-local.
 */
#ifndef PLX_H_
#define PLX_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PLX_API __attribute__((visibility("default")))
#else
#define PLX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum plx_status {
  PLX_OK = 0,
  PLX_ERR_INVALID_ARGUMENT = 1,    /* null/misaligned pointer, bad size      */
  PLX_ERR_UNSUPPORTED = 2,         /* valid request this build cannot run    */
  PLX_ERR_WORKSPACE_TOO_SMALL = 3, /* decode workspace below the query size  */
  PLX_ERR_CUDA = 4                 /* a CUDA runtime call or launch failed   */
} plx_status;

typedef enum plx_dtype { PLX_F32 = 0, PLX_BF16 = 1 } plx_dtype;

/*
 * plx_prefill_fwd -- multi-head / grouped-query Parallax attention forward.
 *
 *   q, rho : [B, L, H_q, d]   queries and probes (one probe per query row)
 *   k, v   : [B, L, H_kv, d]  keys and values
 *   out    : [B, L, H_q, d]   written, in dtype
 *   lse    : [B, H_q, L] fp32, written if non-NULL: natural-log
 *            log-sum-exp of the scaled scores of each row (the softmax
 *            normaliser; independent of rho)
 *   causal : 1 = row i sees keys 0..i; 0 = every row sees all L keys
 *   dtype  : of q, rho, k, v and out
 *   softmax_scale : the score scale (1/sqrt(d) in the textbook form,
 *            page 1 section 1.1); any finite value
 * Sizes: B, L, H_q, H_kv >= 1 (B == 0 or L == 0 is a no-op returning PLX_OK).
 * PLX_BF16 computes S = q.k and t = rho.k from the bf16 inputs on the tensor
 * cores and the two value products in fp16 x fp16 with fp32 accumulation: P
 * and P t are rounded to fp16 (11 significant bits), V is scaled by a power of
 * two per key tile and work unit (block floating point, undone in the
 * epilogue) so that every finite bf16 V keeps 11 significant bits relative to
 * the largest |v| of its tile.  A result that does not fit fp32 sets device
 * error 3 (plx_device_error).
 * Operator definition: page 1 section 1.3 and page 3 (see the file header).
 */
PLX_API plx_status plx_prefill_fwd(const void* q, const void* rho, const void* k,
                                   const void* v, void* out, float* lse, int causal, int B,
                                   int L, int H_q, int H_kv, int d, plx_dtype dtype,
                                   float softmax_scale, void* stream);

/*
 * plx_prefill_fwd_ex -- plx_prefill_fwd with the output dtype chosen apart
 * from the input dtype.
 *
 *   out_dtype : dtype of out; equal to dtype, or PLX_F32 with PLX_BF16 inputs
 *               (the fp32 result before the final rounding to bf16's 8
 *               significant bits)
 * Every other argument, requirement and error as plx_prefill_fwd.  With
 * out_dtype == dtype the call is plx_prefill_fwd.
 */
PLX_API plx_status plx_prefill_fwd_ex(const void* q, const void* rho, const void* k,
                                      const void* v, void* out, float* lse, int causal, int B,
                                      int L, int H_q, int H_kv, int d, plx_dtype dtype,
                                      plx_dtype out_dtype, float softmax_scale, void* stream);

/*
 * plx_prefill_varlen -- plx_prefill_fwd over sequences of different lengths
 * packed along the token axis (same operator per sequence; page 1 opening
 * formula and section 1.3).
 *
 *   q, rho, out : [total_tokens, H_q, d]   k, v : [total_tokens, H_kv, d]
 *   lse         : [H_q, total_tokens] fp32, natural log; may be NULL
 *   cu_seqlens  : [num_seqs + 1] int32, device, 4-byte aligned: sequence s is
 *                 tokens cu_seqlens[s] .. cu_seqlens[s+1]-1 (0 = cu[0] <= cu[1]
 *                 <= ... <= cu[num_seqs] <= total_tokens)
 *   max_seqlen  : an upper bound on every sequence's length (host value)
 * Other arguments as plx_prefill_fwd; a sequence attends only to its own keys
 * (causal: to its own keys up to the query's position).  PLX_BF16 only
 * (PLX_F32 returns PLX_ERR_UNSUPPORTED).  Inconsistent cu_seqlens or a
 * sequence longer than max_seqlen set device error 2 (plx_device_error); rows
 * of such a sequence beyond max_seqlen are not written.  Each sequence's rows
 * equal plx_prefill_fwd on that sequence alone (B = 1, L = its length).
 */
PLX_API plx_status plx_prefill_varlen(const void* q, const void* rho, const void* k,
                                      const void* v, void* out, float* lse,
                                      const int32_t* cu_seqlens, int num_seqs,
                                      int total_tokens, int max_seqlen, int causal, int H_q,
                                      int H_kv, int d, plx_dtype dtype, plx_dtype out_dtype,
                                      float softmax_scale, void* stream);

/*
 * plx_probe_projection -- the probe projection rho = W_R x for a block of
 * tokens (page 1 section 1.3: one extra projection matrix, rho_i = W_R x_i;
 * page 3: the probe is computed from the layer input), as the GEMM
 *
 *     rho[M, N] = x[M, K] W_R[N, K]^T     (fp32 accumulation)
 *
 *   x    : [M, K]  layer inputs, one row per token (K = model width)
 *   w_r  : [N, K]  W_R, row n = output feature n (N = H_q * d for the
 *                  attention's probe layout [.., H_q, d])
 *   rho  : [M, N]  written, in dtype
 * PLX_BF16 runs on the tensor cores and needs K % 8 == 0, N % 8 == 0 and
 * M, N <= 2^31 - 512; PLX_F32 runs on the CUDA cores and needs N <= 1048560
 * (else PLX_ERR_UNSUPPORTED).  M == 0 or N == 0 is a no-op; K >= 1.
 */
PLX_API plx_status plx_probe_projection(const void* x, const void* w_r, void* rho, int M, int N,
                                        int K, plx_dtype dtype, void* stream);

/*
 * plx_prefill_fwd_x -- plx_prefill_fwd with the probes computed from the layer
 * input: rho = x W_R^T (plx_probe_projection with M = B L, N = H_q d,
 * K = d_model), then the attention forward, both on stream.
 *
 *   x   : [B, L, d_model]   w_r : [H_q d, d_model]
 *   rho : [B, L, H_q, d] written (the probes; the backward needs them too)
 * Every other argument as plx_prefill_fwd.  All arguments of both steps are
 * checked before anything is enqueued.
 */
PLX_API plx_status plx_prefill_fwd_x(const void* q, const void* x, const void* w_r,
                                     const void* k, const void* v, void* rho, void* out,
                                     float* lse, int causal, int B, int L, int H_q, int H_kv,
                                     int d, int d_model, plx_dtype dtype, float softmax_scale,
                                     void* stream);

/*
 * plx_prefill_bwd -- gradients of the prefill operator, for training (page 1
 * section 2.3 trains W_R with the rest of the model; the pages print no
 * gradient, so it is derived from the operator of section 1.3):
 *
 *   with g = dLoss/dout, row i, keys j, a_j = softmax_j(scale q.k_j),
 *   t_j = rho.k_j, tbar = sum a t, o = sum a v, c_j = 1 + tbar - t_j:
 *     dv_j += a_j c_j g
 *     dt_j  = a_j (g.o - g.v_j)
 *     ds_j  = a_j (c_j g.v_j + t_j g.o - g.out - tbar g.o)
 *     dq   += scale sum_j ds_j k_j,   drho += sum_j dt_j k_j,
 *     dk_j += scale ds_j q + dt_j rho
 *
 *   q, rho, dout : [B, L, H_q, d] in dtype      k, v : [B, L, H_kv, d]
 *   dq, drho     : [B, L, H_q, d] fp32, written
 *   dk, dv       : [B, L, H_kv, d] fp32, written (summed over the query
 *                  heads that share a KV head)
 *   workspace    : plx_prefill_bwd_workspace_bytes(B, L, H_q) bytes, 16-byte
 *                  aligned, no initialisation needed
 * Other arguments as plx_prefill_fwd.  Neither the forward's output nor its
 * lse is needed: the kernels recompute what they use, the softmax normaliser
 * included, from q, rho, k, v in fp32 (where one key dominates a row, the
 * gradient's a (X - D) terms cancel and would amplify the fp16 rounding that
 * the tensor-core forward's normaliser carries).  bf16 inputs (d = 64 or 128)
 * run two tcgen05 kernels (fp32 accumulation; each gradient operand enters the
 * products as bf16 high and low parts, about 16 significant bits); fp32 inputs
 * run on the CUDA cores with fp32 arithmetic.  Two launches per call.
 */
PLX_API size_t plx_prefill_bwd_workspace_bytes(int B, int L, int H_q);
PLX_API plx_status plx_prefill_bwd(const void* q, const void* rho, const void* k, const void* v,
                                   const void* dout, float* dq, float* drho, float* dk,
                                   float* dv, int causal, int B, int L, int H_q, int H_kv, int d,
                                   plx_dtype dtype, float softmax_scale, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * plx_decode_workspace_bytes -- device workspace that plx_decode needs for the
 * given shape on the CURRENT device (it depends on the device's SM count).
 * Returns 0 for an invalid shape.
 */
PLX_API size_t plx_decode_workspace_bytes(int B, int H_q, int H_kv, int d, int S_max);

/*
 * plx_decode -- single-token Parallax decode over a KV cache (page 3: a KV
 * cache is still required for decoding).
 *
 *   q, rho           : [B, H_q, d]          the new token's queries and probes
 *   k_cache, v_cache : [B, S_max, H_kv, d]  cached keys and values
 *   seqlens          : [B] int32, device    batch b attends to cache rows
 *                      0 .. seqlens[b]-1; values are clamped to [0, S_max];
 *                      a length of 0 writes out = 0 for that batch
 *   out              : [B, H_q, d]          written
 *   workspace        : device memory of at least
 *                      plx_decode_workspace_bytes(...) bytes, 16-byte aligned,
 *                      contents need no initialisation; it must not be used
 *                      by another call that may run concurrently.
 * Rows beyond seqlens[b] (up to S_max) are never used, whatever they hold.
 */
PLX_API plx_status plx_decode(const void* q, const void* rho, const void* k_cache,
                      const void* v_cache, const int32_t* seqlens, void* out, int B, int H_q,
                      int H_kv, int d, int S_max, plx_dtype dtype, float softmax_scale,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * plx_decode_x -- plx_decode with the new token's probes computed from its
 * layer input: rho = x W_R^T (plx_probe_projection with M = B, N = H_q d,
 * K = d_model), then the decode, both on stream.
 *
 *   x   : [B, d_model]   w_r : [H_q d, d_model]
 *   rho : [B, H_q, d] written
 * Every other argument, the workspace rule and the errors as plx_decode.  All
 * arguments of both steps are checked before anything is enqueued.
 */
PLX_API plx_status plx_decode_x(const void* q, const void* x, const void* w_r,
                                const void* k_cache, const void* v_cache, const int32_t* seqlens,
                                void* rho, void* out, int B, int H_q, int H_kv, int d, int S_max,
                                int d_model, plx_dtype dtype, float softmax_scale,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * plx_decode_state -- plx_decode, but instead of out it writes each (b, h)
 * row's softmax state over this cache, so that a key set split into slices
 * (for example a context spread over several GPUs) can be decoded slice by
 * slice and merged with plx_merge_states.
 *
 *   state : [B, H_q, 2d + 4] fp32, device, 16-byte aligned, written; per row
 *           m, l, z, 0, o[d], u[d]: m is the maximum of the scaled scores in
 *           log2 units (softmax_scale * log2(e) * q.k), l = sum 2^(s - m),
 *           z = sum 2^(s - m) (rho.k), o = sum 2^(s - m) v, u = sum 2^(s - m)
 *           (rho.k) v (unnormalised); an empty key set gives m = -inf and
 *           zeros
 * Every other argument as plx_decode (out is not written).
 */
PLX_API plx_status plx_decode_state(const void* q, const void* rho, const void* k_cache,
                                    const void* v_cache, const int32_t* seqlens, float* state,
                                    int B, int H_q, int H_kv, int d, int S_max, plx_dtype dtype,
                                    float softmax_scale, void* workspace,
                                    size_t workspace_bytes, void* stream);

/*
 * plx_merge_states -- out = ((1 + Z/L) O - U) / L from R states of the same
 * rows (log-sum-exp merge: M = max m_r, weights 2^(m_r - M); L, Z, O, U the
 * weighted sums), the one exchange a context split over R slices needs
 * (page 1 section 1.3 operator; the merge is exact up to rounding).
 *
 *   states : [R, B, H_q, 2d + 4] fp32 (plx_decode_state layout), device
 *   out    : [B, H_q, d] in out_dtype (PLX_F32 or PLX_BF16), written; rows
 *            whose R slices are all empty get 0
 */
PLX_API plx_status plx_merge_states(const float* states, int R, void* out, int B, int H_q, int d,
                                    plx_dtype out_dtype, void* stream);

/*
 * plx_decode_paged -- plx_decode over a paged KV cache (page 3: decoding keeps
 * a KV cache; a serving system stores it in fixed-size pages).
 *
 *   k_pages, v_pages : [num_pages, page_size, H_kv, d] page pools (device,
 *                      16-byte aligned)
 *   block_table      : [B, max_pages_per_seq] int32, device, 4-byte aligned:
 *                      position j of batch b is row j % page_size of page
 *                      block_table[b * max_pages_per_seq + j / page_size]
 *   seqlens          : [B] int32, device, clamped to [0, max_pages_per_seq *
 *                      page_size]; entries of block_table past a sequence's
 *                      last page are never read
 *   page_size        : a multiple of 16 (>= 16); num_pages * page_size and
 *                      max_pages_per_seq * page_size below 2^31
 * q, rho, out, workspace, dtype, softmax_scale, stream: as plx_decode (the
 * workspace size is plx_decode_workspace_bytes with S_max =
 * max_pages_per_seq * page_size).  A page index outside [0, num_pages) read
 * for a live position sets device error 2 (plx_device_error) and reads as
 * zeros.  The result is bit-identical to plx_decode on the same rows stored
 * contiguously.
 */
PLX_API plx_status plx_decode_paged(const void* q, const void* rho, const void* k_pages,
                                    const void* v_pages, const int32_t* block_table,
                                    const int32_t* seqlens, void* out, int B, int H_q,
                                    int H_kv, int d, int num_pages, int page_size,
                                    int max_pages_per_seq, plx_dtype dtype, float softmax_scale,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * plx_decode_append -- one serving decode step: append the new token's key and
 * value to the KV cache, then plx_decode over the cache including it (page 3:
 * decoding keeps a KV cache; each step adds the new token's key and value).
 *
 *   k_new, v_new     : [B, H_kv, d] in dtype, device, 16-byte aligned; the new
 *                      token's key and value rows
 *   k_cache, v_cache : [B, S_max, H_kv, d], written: for every batch with
 *                      n = clamp(seqlens[b], 0, S_max) > 0, cache row n - 1
 *                      becomes k_new[b] (resp. v_new[b]); no other row changes
 *   seqlens          : lengths that already count the new token
 * Every other argument, the workspace rule and the errors are those of
 * plx_decode.  All checks run before anything is written; on success two
 * writes happen in stream order: the append (one kernel), then the decode.
 */
PLX_API plx_status plx_decode_append(const void* q, const void* rho, const void* k_new,
                                     const void* v_new, void* k_cache, void* v_cache,
                                     const int32_t* seqlens, void* out, int B, int H_q,
                                     int H_kv, int d, int S_max, plx_dtype dtype,
                                     float softmax_scale, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * plx_decode_static_ws -- plx_decode for callers that cannot allocate device
 * memory.  The pages have no counterpart to this entry point: it is a service
 * of the library.  Callers it serves: a serving loop that must not enter the
 * device allocator on its per-token path (cudaMalloc can synchronise the
 * device and stall), a plugin whose host framework owns the whole device
 * memory pool, or a C caller with no device allocator at hand.
 *
 * Arguments and results are those of plx_decode without the workspace: the
 * caller still passes every input and the output.  The workspace is a fixed
 * 1 MiB array in the library's device memory, present on every GPU that loads
 * the library until the process exits.  The workspace a shape needs is
 * plx_decode_workspace_bytes(...) = 64 + 8 * SMs * (4 + h * (2 d + 4)) bytes,
 * with SMs the device's multiprocessor count and h = 2 if H_q / H_kv is even,
 * else 1; a shape needing more than 1 MiB returns PLX_ERR_WORKSPACE_TOO_SMALL.
 * At d = 128, h = 2 that is 4192 bytes per SM: B200's 148 SMs need 0.59 MiB,
 * and every valid shape fits on any device with up to 250 SMs.  No allocation
 * of any kind.
 *
 * The first call on a device looks up the array's device address with
 * cudaGetSymbolAddress (once per device, with that device current); make that
 * first call before any stream capture.  Every call on a device shares the one
 * array, so calls whose work may overlap on the GPU (different streams, host
 * threads) race on it and must be serialised by the caller.  Its contents
 * carry over between calls; nothing in it needs clearing.
 */
PLX_API plx_status plx_decode_static_ws(const void* q, const void* rho, const void* k_cache,
                                        const void* v_cache, const int32_t* seqlens, void* out,
                                        int B, int H_q, int H_kv, int d, int S_max,
                                        plx_dtype dtype, float softmax_scale, void* stream);

/* Human-readable name of a status code (static storage). */
PLX_API const char* plx_status_string(plx_status s);

/* cudaError_t behind this thread's last PLX_ERR_CUDA (0 if none). */
PLX_API int plx_last_cuda_error(void);

/*
 * plx_device_error -- reads (and, if clear != 0, resets) the device-side error
 * word of the current device: 0 = none, 1 = a bounded wait ran out of time,
 * 2 = a kernel saw inconsistent internal state, 3 = a result was not finite
 * (inputs outside the supported range).  Synchronises the device.
 * Returns PLX_OK or PLX_ERR_CUDA.
 */
PLX_API plx_status plx_device_error(int* code, int clear);

/*
 * plx_set_wait_limit_ns -- diagnostic: the wall-clock limit of every bounded
 * wait in the library's kernels on the current device (default 2 s; ns = 0
 * restores it; otherwise 1000 <= ns <= 6e10).  Meant for tests of the failure
 * detection: a shorter limit makes a stalled wait give up sooner, and a limit
 * shorter than a legitimate stall makes a correct kernel give up and report a
 * timeout.  Synchronises the device.  The pages have no counterpart to this
 * entry point.
 */
PLX_API plx_status plx_set_wait_limit_ns(unsigned long long ns);

/*
 * plx_selftest_wait -- diagnostic: enqueues on stream one warp that waits on a
 * barrier nothing ever completes, through the same bounded wait every kernel of
 * the library uses.  When the limit (plx_set_wait_limit_ns) runs out the kernel
 * records code 1 in the device error word (plx_device_error) and returns; the
 * context stays usable.  Returns PLX_OK once enqueued.  The pages have no
 * counterpart to this entry point.
 */
PLX_API plx_status plx_selftest_wait(void* stream);

/* Library version, major * 10000 + minor * 100 + patch. */
PLX_API int plx_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PLX_H_ */
