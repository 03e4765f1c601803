/*
 * la2.h - C ABI of libla2.so: Lightning Attention-2 causal linear attention
 * on NVIDIA B200 (sm_100a).
 *
 * The operation (article "Lightning Attention-2 新一代注意力机制", section
 * "Lightning Attention-2简介", point 1 and Fig. 2):
 *
 *     O = ((Q K^T) ⊙ M) V
 *
 * with no softmax, M the lower-triangular all-ones mask (diagonal included)
 * when causal = 1, and no mask when causal = 0, in which case the result is
 * the right product O = Q (K^T V). Point 2 (Fig. 3) gives the computation the
 * library follows: each sequence is cut into blocks of `block` rows; inside a
 * block the masked left product is used, across blocks the right product
 * Q_i * KV with a running fp32 state KV += K_i^T V_i.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are dense, contiguous, row-major [B, H, N, d] (q, k, dq, dk) and
 *    [B, H, N, dv] (v, o, dout, dv-gradient). Each (b, h) sequence is
 *    independent. Element type is given by `dt` for every tensor of a call.
 *  - All tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *    aligned. Outputs are overwritten (never accumulated into) and must not
 *    overlap any input. The library allocates no device memory on the call
 *    path: scratch is the caller's `workspace` (256-byte aligned).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream). The return value covers argument validation and
 *    launch errors only; errors raised later on the device are reported by
 *    la2_check().
 *  - B, H or N equal to 0 is an empty problem: LA2_OK, nothing is launched,
 *    pointers may then be NULL. Negative sizes, d or dv < 1, causal not in
 *    {0, 1}, an unknown dtype, a NULL or misaligned pointer, or outputs
 *    overlapping inputs give LA2_ERR_INVALID_ARG.
 *  - Supported shapes. LA2_BF16: d, dv in {64, 128}, block in {64, 128};
 *    d = dv = 128 runs on the tensor cores (tcgen05, fp32 accumulation in
 *    tensor memory, fp32 state), every other bf16 shape on the CUDA-core
 *    kernels (fp32 accumulation and state as well). LA2_F32: any
 *    1 <= d, dv <= 128 and block in {16, 32, 64, 128} whose tiles fit in
 *    shared memory (fp32 CUDA-core path). Anything else gives
 *    LA2_ERR_UNSUPPORTED.
 *  - Thread safety. The compute entry points keep no state between calls
 *    apart from a small cache of work plans (mutex-protected). Three
 *    process-wide settings are test and benchmark hooks, NOT thread-safe:
 *    la2_set_chunk_len, la2_set_spin_limit and the la2_profile_* calls. Set
 *    them before other threads call the library, and leave them at their
 *    defaults (0) in production.
 *  - `block` is the algorithm's block size Bk. N need not be a multiple of
 *    it: the ragged last block is zero-padded on load and not stored.
 *  - Gradients are those of L = <dO, O>; backward needs no saved forward
 *    activations (states are recomputed).
 */
#ifndef LA2_H
#define LA2_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LA2_API __attribute__((visibility("default")))
#else
#define LA2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *la2_stream_t; /* same type as cudaStream_t */

typedef enum {
  LA2_OK = 0,
  LA2_ERR_INVALID_ARG = 1, /* bad pointer, size, flag or alignment            */
  LA2_ERR_UNSUPPORTED = 2, /* valid but unsupported dtype/d/dv/block combo    */
  LA2_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than required         */
  LA2_ERR_CUDA = 4,        /* a CUDA runtime/driver call or launch failed     */
  LA2_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up (la2_check)  */
} la2_status;

typedef enum { LA2_F32 = 0, LA2_BF16 = 1 } la2_dtype;

/*
 * Bytes of workspace a la2_forward (is_backward = 0) or la2_backward
 * (is_backward = 1) call with these arguments needs on the CURRENT device.
 * 0 means no workspace is needed. Returns (size_t)-1 for arguments the call
 * would reject. The size depends on the chunk plan (see la2_set_chunk_len) and
 * on the device's SM count.
 */
LA2_API size_t la2_workspace_size(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv,
                          int causal, int block, la2_dtype dt, int is_backward);

/*
 * Forward: o = ((q k^T) ⊙ M) v (causal = 1) or q (k^T v) (causal = 0).
 * Article section "Lightning Attention-2简介", points 1-3 (Fig. 2, Fig. 3).
 * q, k: [B,H,N,d]; v, o: [B,H,N,dv]; all of type dt. fp32 accumulation.
 */
LA2_API la2_status la2_forward(const void *q, const void *k, const void *v, void *o,
                       int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv,
                       int causal, int block, la2_dtype dt,
                       void *workspace, size_t workspace_bytes, la2_stream_t stream);

/*
 * Backward of L = <dout, o> for the same op (the article names its Algorithm 2
 * but does not print it; the gradients are those of the closed form above):
 *   dq = ((dout v^T) ⊙ M) k,  dk = ((dout v^T) ⊙ M)^T q,  dvv = ((q k^T) ⊙ M)^T dout.
 * q, k, dq, dk: [B,H,N,d]; v, dout, dvv: [B,H,N,dv]. `dout` is the upstream
 * gradient dO; `dvv` receives dV (named so to differ from the size dv).
 */
LA2_API la2_status la2_backward(const void *q, const void *k, const void *v, const void *dout,
                        void *dq, void *dk, void *dvv,
                        int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv,
                        int causal, int block, la2_dtype dt,
                        void *workspace, size_t workspace_bytes, la2_stream_t stream);

/*
 * Grouped K/V heads: GQA, and MQA when Hkv = 1 (cccbook long-context chapter,
 * section on MQA/GQA; mhpn.cn blog, section 3: several query heads share one
 * key/value head). The same op per query head, with query head h of batch b
 * reading K/V head h / (H / Hkv) of batch b:
 *   o[b,h] = ((q[b,h] k[b,h/G]^T) ⊙ M) v[b,h/G],  G = H / Hkv.
 * q, o: [B,H,N,d] / [B,H,N,dv]; k: [B,Hkv,N,d]; v: [B,Hkv,N,dv]; H must be a
 * multiple of Hkv >= 1 (else LA2_ERR_INVALID_ARG). Every other convention as
 * for la2_forward / la2_backward / la2_workspace_size; Hkv = H is exactly those
 * calls. In the backward a K/V head's gradients add up over the query heads
 * that read it: dk [B,Hkv,N,d] and dvv [B,Hkv,N,dv] receive those sums (fp32
 * accumulation, one rounding to the element type); dq is [B,H,N,d].
 */
LA2_API size_t la2_workspace_size_gqa(int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t d,
                                      int64_t dv, int causal, int block, la2_dtype dt,
                                      int is_backward);
LA2_API la2_status la2_forward_gqa(const void *q, const void *k, const void *v, void *o,
                                   int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t d,
                                   int64_t dv, int causal, int block, la2_dtype dt,
                                   void *workspace, size_t workspace_bytes, la2_stream_t stream);
LA2_API la2_status la2_backward_gqa(const void *q, const void *k, const void *v, const void *dout,
                                    void *dq, void *dk, void *dvv, int64_t B, int64_t H,
                                    int64_t Hkv, int64_t N, int64_t d, int64_t dv, int causal,
                                    int block, la2_dtype dt, void *workspace,
                                    size_t workspace_bytes, la2_stream_t stream);

/*
 * Sequence parallelism: one part (a contiguous range of N rows) of longer
 * causal sequences whose other parts live elsewhere, e.g. on other GPUs
 * (youleyou.com article, section "小结": sequence-parallel linear attention as
 * the next step; section "Lightning Attention-2简介", point 2: the part's
 * inter-block term is its queries times the state of everything before it).
 * q, k, v, o, dout, dq, dk, dvv: this part, [B,H,N,.] as for la2_forward
 * (one K/V head per query head). States are fp32, row-major [d][dv] per
 * (b, h), device memory, 16-byte aligned:
 *  - prefix_states [n_prefix][B][H][d][dv]: their sum is the KV state
 *    sum k_t^T v_t of every token before this part (la2_kv_state of each
 *    earlier part);
 *  - suffix_states [n_suffix][B][H][d][dv]: their sum is sum q_t^T dO_t over
 *    every token after this part (la2_kv_state with (q, dO) in the (k, v)
 *    slots, for each later part).
 * la2_forward_sp writes the part's causal output o_t = q_t P + sum over the
 * part's s <= t of (q_t . k_s) v_s; la2_backward_sp the part's gradients of
 * the whole sequence's L = <dO, O> (dq += dO P^T, dk += v U^T, dv += k U for
 * the summed prefix P and suffix U). n = 0 means no such parts (NULL allowed);
 * states must not overlap the outputs. Workspace: la2_workspace_size_sp.
 * Other conventions and errors as for la2_forward / la2_backward.
 */
LA2_API size_t la2_workspace_size_sp(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv,
                                     int block, la2_dtype dt, int is_backward);
LA2_API la2_status la2_forward_sp(const void *q, const void *k, const void *v, void *o,
                                  const float *prefix_states, int64_t n_prefix, int64_t B,
                                  int64_t H, int64_t N, int64_t d, int64_t dv, int block,
                                  la2_dtype dt, void *workspace, size_t workspace_bytes,
                                  la2_stream_t stream);
LA2_API la2_status la2_backward_sp(const void *q, const void *k, const void *v, const void *dout,
                                   void *dq, void *dk, void *dvv, const float *prefix_states,
                                   int64_t n_prefix, const float *suffix_states, int64_t n_suffix,
                                   int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv, int block,
                                   la2_dtype dt, void *workspace, size_t workspace_bytes,
                                   la2_stream_t stream);

/*
 * Decayed causal form (a reading: the article gives no decay; its pages mention
 * data-dependent gating only, for gated linear attention). Per query head h a
 * rate lambda[h] multiplies the KV state before each token:
 *   KV_t = lambda KV_{t-1} + k_t^T v_t,   o_t = q_t KV_t,
 * i.e. o = ((q k^T) ⊙ D) v with D[t][s] = lambda^(t-s) for s <= t, 0 above;
 * lambda = 1 is la2_forward's causal op. `lambda`: H fp32 rates in [0, 1],
 * device memory, 4-byte aligned, read only (powers are taken with powf; rates
 * outside [0, 1] are not rejected and follow the same formula). One K/V head per
 * query head; q, k, v, o, dout, dq, dk, dvv as for la2_forward / la2_backward
 * (causal only). At bf16 d = dv = 128 (block 64 or 128) both directions run
 * on tensor cores: the forward as the chunk kernels with decayed chunk states;
 * the backward as three such forwards, dQ from (dO, V, K) and dK, dV from
 * time-reversed copies of q, k, v, dout kept in the workspace (B*H*N at most
 * 2^31 - 1, else LA2_ERR_UNSUPPORTED). Every other shape and dtype la2_forward
 * takes runs on CUDA cores, with the shared-memory limits of that path (f32
 * d = dv = 128 at block 128 does not fit the backward: LA2_ERR_UNSUPPORTED).
 * Workspace: la2_workspace_size_decay; it must not overlap the inputs, the
 * outputs or `lambda`. Other conventions and errors as for la2_forward /
 * la2_backward; `lambda` must not overlap the outputs.
 */
LA2_API size_t la2_workspace_size_decay(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv,
                                        int block, la2_dtype dt, int is_backward);
LA2_API la2_status la2_forward_decay(const void *q, const void *k, const void *v, void *o,
                                     const float *lambda, int64_t B, int64_t H, int64_t N,
                                     int64_t d, int64_t dv, int block, la2_dtype dt,
                                     void *workspace, size_t workspace_bytes, la2_stream_t stream);
LA2_API la2_status la2_backward_decay(const void *q, const void *k, const void *v,
                                      const void *dout, void *dq, void *dk, void *dvv,
                                      const float *lambda, int64_t B, int64_t H, int64_t N,
                                      int64_t d, int64_t dv, int block, la2_dtype dt,
                                      void *workspace, size_t workspace_bytes,
                                      la2_stream_t stream);

/*
 * Synchronises `stream`, then reports and clears the device-side error word
 * that kernels set when a bounded wait gives up (LA2_ERR_TIMEOUT), or
 * LA2_ERR_CUDA if the stream holds a CUDA error. LA2_OK otherwise.
 */
LA2_API la2_status la2_check(la2_stream_t stream);

/* Static, human-readable name of a status code. */
LA2_API const char *la2_status_string(la2_status s);

/*
 * Work split override, a test hook. 0 (the default) lets the library split
 * the work from B*H, N and the SM count (see la2_plan_ranges). A positive
 * value cuts every sequence into chunks of `chunk_len` rows (rounded up to a
 * multiple of `block`) that run in parallel from the sum of the earlier
 * chunks' KV states (a sum, so any split gives the same result up to fp32
 * rounding order). Process-wide and not thread-safe: it changes the plan and
 * la2_workspace_size of every later call from any thread. A forced split of the
 * tensor-core causal path into more than 160 chunks in total runs on the
 * chunk kernels instead of the persistent range split (same results; the
 * workspace size accounts for it). Returns LA2_ERR_INVALID_ARG for a
 * negative value.
 */
LA2_API la2_status la2_set_chunk_len(int64_t chunk_len);

/*
 * Work split the next call with these arguments uses. The (b, h) sequences are
 * laid end to end as B*H*ceil(N/block) blocks; the call runs R ranges of that
 * list in parallel, range r covering blocks [starts[r], starts[r+1]). A range
 * that starts inside a sequence starts from the KV state of that sequence's
 * earlier blocks. Returns R and, when cap >= R + 1, writes the R + 1 starts;
 * returns -1 for arguments the call would reject.
 */
LA2_API int64_t la2_plan_ranges(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv,
                                int causal, int block, la2_dtype dt, int is_backward,
                                int64_t *starts, int64_t cap);

/*
 * Inference form (article, section "Lightning Attention-2速度对比": linear
 * attention converts losslessly to an RNN; section "Lightning Attention-2简介",
 * point 2: the KV state carried from block to block). A per-sequence state
 * S is d x dv fp32, row-major; `state` is [B, H, d, dv] fp32 device memory
 * owned by the caller, 16-byte aligned, updated in place.
 *
 * la2_kv_state: the state a prefill leaves, S += sum_t k_t^T v_t over the N
 * tokens of each sequence (pass a zeroed state for a fresh sequence; a later
 * call continues it). k [B,H,N,d], v [B,H,N,dv] in `dt`; shapes as for
 * la2_forward with block 64. Scratch: la2_kv_state_workspace_size() bytes of
 * `workspace` (256-byte aligned; (size_t)-1 for an invalid shape). The per-chunk
 * states are summed in a fixed order, so repeated calls give identical bits.
 * Errors as for la2_forward; `state` must not overlap k, v or the workspace.
 */
LA2_API size_t la2_kv_state_workspace_size(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv,
                                           la2_dtype dt);
LA2_API la2_status la2_kv_state(const void *k, const void *v, float *state, int64_t B, int64_t H,
                                int64_t N, int64_t d, int64_t dv, la2_dtype dt, void *workspace,
                                size_t workspace_bytes, la2_stream_t stream);

/*
 * la2_decode_step: one new token per sequence in RNN form,
 *     S += k^T v,   o = q S
 * (the token's own pair counts, as the diagonal of the causal mask does).
 * q, k [B,H,d], v, o [B,H,dv] in `dt` (aligned to their element size), state
 * as above. Any d, dv >= 1 and both dtypes; fp32 arithmetic. Continuing from
 * la2_kv_state over tokens 0..N-1, step t gives row t of la2_forward's causal
 * output. o must not overlap any input or the state; B or H = 0 is empty.
 */
LA2_API la2_status la2_decode_step(const void *q, const void *k, const void *v, void *o,
                                   float *state, int64_t B, int64_t H, int64_t d, int64_t dv,
                                   la2_dtype dt, la2_stream_t stream);

/*
 * Upper bound, in spin iterations, of every device-side wait (mbarrier or
 * flag). When a wait exceeds it the kernel records LA2_ERR_TIMEOUT in the
 * device error word, stops its work and returns; la2_check() reports it.
 * 0 restores the default (large enough to be reached only by a fault).
 * Process-wide test hook, not thread-safe.
 */
LA2_API la2_status la2_set_spin_limit(int64_t iterations);

/*
 * Per-kernel launch timing, for benchmarks. While enabled, every kernel the
 * library launches is bracketed by a pair of CUDA events on its stream.
 * la2_profile_enable(1) clears the records and starts recording, (0) pauses,
 * (2) resumes without clearing (so a benchmark can time a sample of its
 * steps); other values give LA2_ERR_INVALID_ARG. la2_profile_collect()
 * synchronises the events and returns, for kernel id `kernel`, the number of
 * recorded launches and their summed device time in ms since the last
 * la2_profile_enable(1). Ids run from 0 to la2_profile_num_kernels()-1 and
 * la2_profile_kernel_name() names them. Process-wide benchmark hook, not
 * thread-safe: while enabled, the launches of every thread are recorded.
 */
LA2_API la2_status la2_profile_enable(int on);
LA2_API int la2_profile_num_kernels(void);
LA2_API const char *la2_profile_kernel_name(int kernel);
LA2_API la2_status la2_profile_collect(int kernel, int64_t *launches, double *total_ms);

/*
 * la2_forward_noalloc: la2_forward without a workspace argument. The article
 * has no counterpart; this entry point exists for callers that cannot
 * allocate device memory at the time they call the op (for example an
 * operator hosted by a runtime that owns all device memory and offers no
 * scratch space, or a serving loop that forbids allocations after start-up).
 *
 * The chunk states that la2_forward keeps in the caller's workspace live here
 * in one array of LA2_NOALLOC_SCRATCH_BYTES (32 MiB) compiled into the
 * library: every GPU on which the library is loaded holds that memory until
 * the process exits. The first call on each device looks up the array's
 * device address (cudaGetSymbolAddress, with that device current); make that
 * first call before any stream capture. A problem whose workspace
 * (la2_workspace_size(..., is_backward = 0)) exceeds the array returns
 * LA2_ERR_WORKSPACE without launching anything; other arguments and errors are
 * as for la2_forward. The call allocates nothing.
 *
 * All calls share the one array and it keeps the previous call's contents
 * (every element a call reads it first writes). Calls that may overlap on the
 * GPU - on different streams, or from host threads without ordering between
 * them - race on the array and give wrong results: serialise them.
 */
#define LA2_NOALLOC_SCRATCH_BYTES (32u << 20)
LA2_API la2_status la2_forward_noalloc(const void *q, const void *k, const void *v, void *o,
                                       int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv,
                                       int causal, int block, la2_dtype dt, la2_stream_t stream);

/* Library version, (major << 16) | minor. */
LA2_API int la2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LA2_H */
