/*
 * hh.h -- C ABI of libhh.so, the B200 (sm_100a) kernels of a hybrid
 * linear / full attention layer.
 *
 * The layer is the one the pages describe:
 *  - "The Hybrid Attention in Qwen3.8-27B -- Only 16 of 64 Layers Grow a KV
 *    Cache": 16 x (3 x Gated DeltaNet -> 1 x Gated Attention); the Gated
 *    DeltaNet side has 48 value heads over 16 q/k heads at head dim 128, the
 *    attention side 24 query heads over 4 key/value heads at head dim 256
 *    (sections "Why 27B parameters can carry 262K tokens" and "Grouped-query
 *    attention multiplies on top of that").
 *  - "The economics of hybrid attention": the linear layers keep a fixed-size
 *    recurrent state (TL;DR), the attention layers a KV cache that grows per
 *    token ("What a token of context costs").
 *  - "HydraHead: From Head-Level Functional Heterogeneity to Specialized
 *    Attention Hybridization", abstract: softmax-attention heads (FA) and
 *    linear heads (LA) side by side in one layer, whose outputs meet in a
 *    scale-normalized fusion module.
 *  - "PHBA: Prefix-State Hybrid Block Attention", abstract and Figure 1: top-K
 *    block retrieval whose blocks come with prefix states, one softmax over
 *    the retrieved tokens and the state slots.
 * The pages print no formula.  The arithmetic implemented here is the plain
 * reading stated at each entry point.
 *
 * Conventions for every entry point
 *  - bf16 tensors are passed as hh_bf16 (the raw 16-bit pattern).
 *  - All tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *    aligned, contiguous in the stated layout (last index fastest), except
 *    head_is_fa of hybrid_head_layer_fwd, which is a HOST array.
 *  - Work is enqueued on `stream` (NULL = legacy default stream) and is
 *    asynchronous.  The library never allocates device memory on these calls;
 *    scratch comes from the caller through the *_workspace_size queries.
 *  - Arguments are validated before anything is enqueued.  On any error the
 *    call returns a negative status, enqueues nothing and leaves every output
 *    untouched; hh_last_error() then describes the error (thread-local).
 *  - Outputs must not alias inputs (except the in-place state of
 *    gdn_decode_step).  The library keeps no state between calls other than
 *    the thread-local error string and one device status word, so calls on
 *    different streams may run concurrently.
 */
#ifndef HH_H_
#define HH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define HH_API __attribute__((visibility("default")))
#else
#define HH_API
#endif

typedef uint16_t hh_bf16;
typedef struct CUstream_st *hh_stream;

enum {
  HH_OK = 0,
  HH_ERR_INVALID_ARG = -1, /* null pointer, bad size, misaligned pointer, bad layout */
  HH_ERR_UNSUPPORTED = -2, /* a valid request this build has no kernel for (e.g. d=64) */
  HH_ERR_CUDA = -3,        /* a CUDA runtime call failed (launch or query) */
  HH_ERR_TIMEOUT = -4      /* a device-side bounded wait gave up (see hh_device_status) */
};

/* Description of the last error on the calling thread ("" if none).  The
 * pointer stays valid until the next library call on that thread. */
HH_API const char *hh_last_error(void);

/* Version string of the library build. */
HH_API const char *hh_version(void);

/* Synchronises `stream`, then returns and clears the device status word:
 * HH_OK, or HH_ERR_TIMEOUT if a kernel's bounded wait expired since the last
 * query (the kernel then skipped its remaining work and exited cleanly), or
 * HH_ERR_CUDA if the synchronisation itself failed. */
HH_API int hh_device_status(hh_stream stream);

/* Failure-path self-test: enqueues a one-thread kernel that waits on a
 * barrier nothing ever arrives on, bounded by `limit_us` microseconds
 * (1 .. 2,000,000).  The expiry sets the device status word exactly as an
 * expired wait in any other kernel would, so the next hh_device_status() on
 * the stream returns HH_ERR_TIMEOUT.  Nothing faults, traps or hangs. */
HH_API int hh_selftest_wait_timeout(unsigned limit_us, hh_stream stream);

/*
 * gdn_chunk_fwd -- gated delta rule over a whole sequence (prefill).
 *
 * Per sequence b and value head h, with q/k head hq = h / (H_v / H_qk)
 * (contiguous groups), starting from S_0 = state_in[b,h] (or zeros), for
 * t = 0 .. T-1:
 *     S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = scale * S_t q_t
 * S is d_v x d_k, fp32.  The pages name the layer (Gated DeltaNet, a fixed-size
 * state per head: "The Hybrid Attention in Qwen3.8-27B", section "Why 27B
 * parameters can carry 262K tokens"; its head counts, section "Grouped-query
 * attention multiplies on top of that") but print no formula; this is the
 * plain reading.
 * Evaluated in chunks of `chunk` tokens, in two passes: the state-free part
 * of every chunk (K K^T, Q K^T, the triangular inverse of the WY/UT form in
 * fp32, its products with K and V, and the state-free part of the output map)
 * for all chunks in parallel into `workspace`, then the sequential scan over
 * chunks that carries the fp32 state, one affine update S <- gamma_C S - S M + B
 * per chunk.  5th-generation tensor cores (tcgen05, accumulators in tensor
 * memory) with bf16 operands and fp32 accumulation; the state stays fp32.
 *
 *   q, k       [B, T, H_qk, d_k]  bf16
 *   v, o       [B, T, H_v, d_v]   bf16   (o written)
 *   g, beta    [B, T, H_v]        fp32   (g = log of the per-token decay)
 *   state_in   [B, H_v, d_v, d_k] fp32   nullable: zeros
 *   state_out  [B, H_v, d_v, d_k] fp32   nullable: not written; may equal
 *                                        state_in (in-place update)
 *   workspace  device scratch of gdn_chunk_fwd_workspace_size(B, T, H_v, d_v,
 *              chunk) bytes, 256-byte aligned (56.5 KB per value head and
 *              chunk of 64 tokens); contents on entry are ignored.  May be
 *              NULL when T = 0.
 * Supported: d_k = d_v = 128, chunk = 64, H_v % H_qk == 0, B >= 1, T >= 0
 * (any T up to 4194240; a last partial chunk is masked).  T = 0 copies
 * state_in to state_out.
 * When B * H_v is at most half the SM count, the state-free pass and the scan
 * run side by side on two library-owned streams (the scan at the device's
 * highest stream priority, the state-free pass one step below), the scan's
 * CTAs waiting (bounded) for each chunk's record; the call is joined back into
 * `stream`.  Calls issued
 * concurrently on different streams must together keep those waiting scans
 * under the SM count, else their waits expire with HH_ERR_TIMEOUT.
 */
HH_API size_t gdn_chunk_fwd_workspace_size(int B, int T, int H_v, int d_v, int chunk);
HH_API int gdn_chunk_fwd(const hh_bf16 *q, const hh_bf16 *k, const hh_bf16 *v, const float *g,
                         const float *beta, const float *state_in, float *state_out, hh_bf16 *o,
                         void *workspace, size_t ws_bytes, int B, int T, int H_qk, int H_v,
                         int d_k, int d_v, float scale, int chunk, hh_stream stream);

/*
 * gdn_chunk_bwd -- gradients of gdn_chunk_fwd (the backward pass of a Gated
 * DeltaNet layer).  The pages say the hybrid heads are trained (the HydraHead
 * abstract's transfer and distillation pipeline; PHBA's Figure 3, training
 * throughput) but print no formula; this is the plain reading: with output
 * cotangents dO and dstate_out (the cotangent of S_T, nullable: zero), the
 * gradients of  L = sum_t o_t . dO_t + S_T . dstate_out  with respect to q, k,
 * v, g, beta and S_0, through the recurrence of gdn_chunk_fwd.
 * Chunked: the forward pass keeps every chunk's start state, a reverse scan over
 * chunks carries the state's cotangent (dS_c = dS_{c+1} A_c^T + scale dO_c^T Qt_c
 * for the chunk map S_{c+1} = S_c A_c + B_c), and every chunk then pulls the
 * cotangents of its maps back through the WY solve and the decay masks to its
 * tokens.  Values stay fp32; the products run on the tensor cores with each
 * fp32 operand split into two bf16 terms (fp32-accurate).
 *
 *   q, k, v, g, beta, state_in   as for gdn_chunk_fwd (state_in nullable)
 *   dO          [B, T, H_v, d_v]   bf16
 *   dstate_out  [B, H_v, d_v, d_k] fp32  nullable (zero)
 *   dq, dk      [B, T, H_qk, d_k]  fp32  written (summed over the value heads
 *                                        sharing a q/k head)
 *   dv          [B, T, H_v, d_v]   fp32  written
 *   dg, dbeta   [B, T, H_v]        fp32  written
 *   dstate_in   [B, H_v, d_v, d_k] fp32  nullable: the gradient of S_0
 *   workspace   gdn_chunk_bwd_workspace_size(B, T, H_v, d_v, chunk) bytes,
 *               256-byte aligned: the forward records and output, the chunk
 *               start states, their cotangents and the chunk maps (about 264 KB
 *               per value head and chunk), and up to 296 x 720 KB of per-CTA
 *               scratch (at most 218 MB).
 * Supported: d_k = d_v = 128, chunk = 64, H_v % H_qk == 0, B >= 1, T >= 1.
 */
HH_API size_t gdn_chunk_bwd_workspace_size(int B, int T, int H_v, int d_v, int chunk);
HH_API int gdn_chunk_bwd(const hh_bf16 *q, const hh_bf16 *k, const hh_bf16 *v, const float *g,
                         const float *beta, const float *state_in, const hh_bf16 *dO,
                         const float *dstate_out, float *dq, float *dk, float *dv, float *dg,
                         float *dbeta, float *dstate_in, void *workspace, size_t ws_bytes, int B,
                         int T, int H_qk, int H_v, int d_k, int d_v, float scale, int chunk,
                         hh_stream stream);

/*
 * gdn_decode_step -- one token of the gated delta rule per sequence, updating
 * the state in place: the decode form of gdn_chunk_fwd with T = 1.  The cost
 * of a decode token in these layers is the state, read and written once,
 * whatever the context length ("The economics of hybrid attention", TL;DR).
 * One pass over each state: every fp32 element is read once and written once.
 *
 *   q, k    [B, H_qk, d_k]       bf16
 *   v, o    [B, H_v, d_v]        bf16  (o written)
 *   g, beta [B, H_v]             fp32
 *   state   [B, H_v, d_v, d_k]   fp32  read and overwritten with S_1
 * Supported: d_k = d_v = 128, H_v % H_qk == 0, B >= 1.
 */
HH_API int gdn_decode_step(const hh_bf16 *q, const hh_bf16 *k, const hh_bf16 *v, const float *g,
                    const float *beta, float *state, hh_bf16 *o, int B, int H_qk, int H_v,
                    int d_k, int d_v, float scale, hh_stream stream);

/*
 * gqa_attn_fwd -- grouped-query softmax attention over a whole sequence
 * (prefill), with an optional sigmoid output gate ("Gated Attention": "The
 * Hybrid Attention in Qwen3.8-27B", section "Grouped-query attention
 * multiplies on top of that", 24 query heads over 4 key/value heads).
 *
 * For query head h (key/value head hk = h / (H_q / H_kv), contiguous groups)
 * and position t:   o_t = sum_{j in J(t)} softmax_j(scale * q_t . k_j) v_j,
 * J(t) = {0..t} if causal, else {0..T-1};  then, if gate != NULL,
 * o_t <- o_t * sigmoid(gate_t) elementwise.  fp32 accumulation and softmax.
 *
 *   q, gate, o [B, T, H_q, d]  bf16   (gate nullable; o written)
 *   k, v       [B, T, H_kv, d] bf16
 * Supported: d in {128, 256}, H_q % H_kv == 0, B >= 1, T >= 0.
 */
HH_API int gqa_attn_fwd(const hh_bf16 *q, const hh_bf16 *k, const hh_bf16 *v, const hh_bf16 *gate,
                 hh_bf16 *o, int B, int T, int H_q, int H_kv, int d, float scale, int causal,
                 hh_stream stream);

/*
 * gqa_attn_decode -- one new query per sequence against its KV cache
 * (split over the cache, partial softmax statistics merged by log-sum-exp).
 * The cache is the per-token cost of the attention layers ("The economics of
 * hybrid attention", section "What a token of context costs").
 * The cache already holds the current token; nothing is appended.
 *
 *   q, gate, o         [B, H_q, d]          bf16  (gate nullable; o written)
 *   k_cache, v_cache   [B, T_cache, H_kv, d] bf16
 *   cache_len          [B] int32 device array, nullable (all = T_cache);
 *                      sequence b attends positions 0 .. cache_len[b]-1,
 *                      values are clamped to [0, T_cache]; a sequence with
 *                      length 0 gets a zero output row.
 *   workspace          device scratch of at least
 *                      gqa_attn_decode_workspace_size(B, H_q, d, T_cache) bytes
 *                      (256-byte aligned); contents on entry are ignored.
 * Supported: d = 256 or 128, H_q % H_kv == 0, H_q / H_kv <= 16, B >= 1.
 */
HH_API size_t gqa_attn_decode_workspace_size(int B, int H_q, int d, int T_cache);
HH_API int gqa_attn_decode(const hh_bf16 *q, const hh_bf16 *k_cache, const hh_bf16 *v_cache,
                    const int32_t *cache_len, const hh_bf16 *gate, hh_bf16 *o, void *workspace,
                    size_t ws_bytes, int B, int T_cache, int H_q, int H_kv, int d, float scale,
                    hh_stream stream);

/*
 * gqa_attn_decode_q8_0 -- gqa_attn_decode over a KV cache kept in the q8_0
 * format that "The economics of hybrid attention" chooses for long contexts
 * (table in "What a token of context costs": 34 KiB per token for the 16
 * attention layers, against 64 KiB in f16; section "Why q8, not q4").  Each
 * block of 32 consecutive elements of a cached K or V row is 32 int8 values
 * x_i and one fp16 scale s and stands for s * x_i.  The pages give the format's
 * size only; this library's layout keeps values and scales in two arrays (same
 * bytes per token as the interleaved 34-byte blocks, with aligned vector loads).
 * The cache is dequantised in registers; the result is the attention of
 * gqa_attn_decode over the dequantised cache.
 *
 *   q, gate, o           [B, H_q, d]             bf16  (gate nullable; o written)
 *   k_values, v_values   [B, T_cache, H_kv, d]   int8
 *   k_scales, v_scales   [B, T_cache, H_kv, d/32] fp16 bit patterns, 16-byte aligned
 *   cache_len, workspace as for gqa_attn_decode (the same workspace size query).
 * Supported: d = 256, H_q % H_kv == 0, H_q / H_kv <= 16, B >= 1.
 */
HH_API int gqa_attn_decode_q8_0(const hh_bf16 *q, const int8_t *k_values, const uint16_t *k_scales,
                                const int8_t *v_values, const uint16_t *v_scales, const int32_t *cache_len,
                                const hh_bf16 *gate, hh_bf16 *o, void *workspace, size_t ws_bytes, int B,
                                int T_cache, int H_q, int H_kv, int d, float scale, hh_stream stream);

/*
 * gqa_attn_decode_noalloc/*
 * gqa_attn_decode_noalloc -- gqa_attn_decode for callers that cannot allocate.
 * The pages have no counterpart of this entry point; it exists for callers
 * that are handed only their input and output buffers (for example a plugin
 * inside a host framework that gives it no allocator) or that must not call
 * cudaMalloc / cudaFree per step, since those can synchronise the device.
 *
 * Same arguments, layouts and results as gqa_attn_decode, minus the workspace:
 * the scratch is a fixed array of HH_NOALLOC_SCRATCH_BYTES inside the library,
 * held by every GPU that loads the library until the process exits.  Nothing
 * is allocated by this call.  The first call on a device looks up the array's
 * device address (once per device, with that device current), so make that
 * first call before any stream capture.  All calls on a device share the
 * array and it keeps the last call's contents (nothing in it needs to start at
 * zero); calls whose GPU work overlaps (other streams, other host threads)
 * race on it and must be serialised by the caller.
 * Returns HH_ERR_UNSUPPORTED, with a message, when the shape needs more than
 * HH_NOALLOC_SCRATCH_BYTES, i.e. when gqa_attn_decode_workspace_size(B, H_q, d,
 * T_cache) exceeds it (B = 64, H_q = 24, d = 256 and a 131,072-token cache
 * need about 25 MiB).
 */
#define HH_NOALLOC_SCRATCH_BYTES (32u << 20)
HH_API int gqa_attn_decode_noalloc(const hh_bf16 *q, const hh_bf16 *k_cache, const hh_bf16 *v_cache,
                                   const int32_t *cache_len, const hh_bf16 *gate, hh_bf16 *o, int B,
                                   int T_cache, int H_q, int H_kv, int d, float scale,
                                   hh_stream stream);

/*
 * hybrid_head_layer_fwd -- head-level LA/FA hybrid layer ("HydraHead: From
 * Head-Level Functional Heterogeneity to Specialized Attention Hybridization",
 * abstract: FA and LA heads in one layer, joined by scale-normalized fusion).
 *
 * Each of the H heads (head dim d) is either FA (head_is_fa[h] != 0): causal
 * softmax attention with its own K/V, scale_fa, no gate; or LA: the gated
 * delta rule of gdn_chunk_fwd with its own q/k (group size 1), scale_la, and
 * state_in[b,h] (nullable: zeros).  The scale-normalized fusion module has no
 * formula on the pages; this library's fixed choice is an RMS normalisation
 * per (token, head), no learnable gain:
 *     y = x / sqrt(mean_i x_i^2 + eps)         (computed in fp32)
 * and the heads are concatenated: out[b, t, h*d + i] = y_i.  Both paths apply
 * it to the fp32 result before the single bf16 rounding; the LA heads' output
 * product then takes the state as two bf16 terms (hi + lo), since normalising
 * a row of small norm scales up its absolute error.
 * The LA heads are launched first, on `stream`; the FA heads follow on a
 * library-owned stream behind a fork event and are joined back into `stream`.
 *
 *   q, k, v     [B, T, H, d]  bf16
 *   g, beta     [B, T, H]     fp32  (read for LA heads only)
 *   head_is_fa  [H]           uint8 HOST array
 *   state_in    [B, H, d, d]  fp32  nullable (LA entries read)
 *   state_out   [B, H, d, d]  fp32  nullable (LA entries written, FA untouched)
 *   out         [B, T, H*d]   bf16  written
 *   workspace   hybrid_head_layer_workspace_size(B, T, H, d) bytes, 256-byte
 *               aligned (the delta-rule heads' scratch, as for gdn_chunk_fwd)
 * Supported: d = 128, chunk = 64, 1 <= H <= 64, B >= 1, 0 <= T <= 4194240.
 */
HH_API size_t hybrid_head_layer_workspace_size(int B, int T, int H, int d);
HH_API int hybrid_head_layer_fwd(const hh_bf16 *q, const hh_bf16 *k, const hh_bf16 *v, const float *g,
                          const float *beta, const uint8_t *head_is_fa, const float *state_in,
                          float *state_out, hh_bf16 *out, void *workspace, size_t ws_bytes,
                          int B, int T, int H, int d, float scale_la, float scale_fa, float eps,
                          int chunk, hh_stream stream);

/*
 * PHBA ("PHBA: Prefix-State Hybrid Block Attention", abstract and Figure 1):
 * top-K block retrieval whose every retrieved block comes with a prefix state
 * summarising the context before it, and one softmax over the retrieved tokens
 * and the state slots.  The page prints no formula; the plain reading
 * implemented here, per sequence and head, with blocks of C tokens (token t
 * in block t / C, nb = ceil(T / C) blocks):
 *
 * phba_prefix_states -- the prefix states (the page builds them with a gated
 * recurrence evaluated at the block edges, over M = 128 memory slots): the
 * gated slot memory
 *     Kt_{t+1}[m] = a_{t,m} Kt_t[m] + (1 - a_{t,m}) k_raw_t
 *     Vt_{t+1}[m] = a_{t,m} Vt_t[m] + (1 - a_{t,m}) v_t,    Kt_0 = Vt_0 = 0,
 * and entry j of the output is the memory after the jC tokens before block j
 * (entry 0 is zero).  Each block's contribution from zero is a product on the
 * tensor cores with fp32 accumulation; the entries are chained in fp32 and
 * rounded to bf16 once.
 *
 *   k_raw, v       [B, T, H, d]       bf16  (d = 128)
 *   alpha          [B, T, H, M]       fp32  slot forget gates in (0, 1)
 *   kstate, vstate [B, H, nb, M, d]   bf16  written
 *   workspace      phba_prefix_states_workspace_size(...) bytes, 256-byte
 *                  aligned (fp32 block contributions: 128 KiB per block and head)
 * Supported: d = M = 128, C in {64, 128, 256}, B, H >= 1, 1 <= T, B H nb M < 2^31.
 */
HH_API size_t phba_prefix_states_workspace_size(int B, int T, int H, int d, int M, int C);
HH_API int phba_prefix_states(const hh_bf16 *k_raw, const hh_bf16 *v, const float *alpha, hh_bf16 *kstate,
                              hh_bf16 *vstate, void *workspace, size_t ws_bytes, int B, int T, int H, int d,
                              int M, int C, hh_stream stream);

/*
 * phba_fwd -- routing and attention (Figure 1: the rotated query routes and
 * reads the retrieved tokens, the raw query reads their prefix states).
 *   routing: query t scores every earlier block j < t / C by
 *     q_rope_t . mean_{s in block j} k_rope_s  (fp32) and keeps the
 *     min(K, t / C) best; a tie goes to the lower block index.
 *   attention: one softmax, logits times scale, over
 *     - every token s of each kept block and the tokens s <= t of the own
 *       block t / C: logit q_rope_t . k_rope_s, value v_s;
 *     - the M slots of the prefix state of each kept block and of the own
 *       block, except block 0's (empty): logit q_raw_t . Kt[m], value Vt[m].
 * Queries are grouped by block into tiles of 128 (the own block's queries
 * with a causal mask, then every query that kept it); each tile runs on the
 * tensor cores and leaves a partial output and log-sum-exp per query, which a
 * last kernel merges.  fp32 accumulation and softmax, bf16 output.
 *
 *   q_rope, k_rope, q_raw, v  [B, T, H, d]      bf16
 *   kstate, vstate            [B, H, nb, M, d]  bf16 (phba_prefix_states)
 *   o                         [B, T, H, d]      bf16  written
 *   sel                       [B, T, H, K]      int32 nullable: written with the
 *                             kept blocks, ascending, -1 after the last
 *   workspace                 phba_fwd_workspace_size(...) bytes, 256-byte
 *                             aligned (about (K + 1) x 264 bytes per query and head)
 * Supported: d = M = 128, C in {64, 128, 256}, 0 <= K <= 16, T / C <= 512,
 * B, H >= 1, T >= 1, B T H (K + 1) < 2^31.
 */
HH_API size_t phba_fwd_workspace_size(int B, int T, int H, int d, int M, int C, int K);
HH_API int phba_fwd(const hh_bf16 *q_rope, const hh_bf16 *k_rope, const hh_bf16 *q_raw, const hh_bf16 *v,
                    const hh_bf16 *kstate, const hh_bf16 *vstate, hh_bf16 *o, int32_t *sel, void *workspace,
                    size_t ws_bytes, int B, int T, int H, int d, int M, int C, int K, float scale,
                    hh_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* HH_H_ */
