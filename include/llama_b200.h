/*
 * llama_b200.h -- C ABI of the B200 (sm_100a) forward pass of the LLaMA
 * pre-norm decoder stack.
 *
 * What is computed (the pages, cited by title and section):
 *   [PFD] "LLaMA: Open and Efficient Foundation Language Models"
 *         (paperfordummies.in), section "The one formula":
 *             h = x + Attn(RMSNorm(x))
 *             y = h + Wdown(SiLU(Wgate RMSNorm(h)) (.) Wup RMSNorm(h))
 *         stacked L times, then one final RMSNorm and an untied output head
 *         producing (n, vocab) logits; no bias anywhere; no position signal
 *         at the bottom.
 *   [PFD] "RMSNorm: LayerNorm minus the mean"; [NAR] "LLaMA: No
 *         Architecture Revolution, Yet It Became the Open-Model
 *         Foundation", section "An Architecture Recipe Without an Invention
 *         Myth": RMSNorm(x) = x / sqrt(mean(x^2) + eps) (.) g.
 *   [PFD] "RoPE: rotate Q and K, leave V alone": Q and K rotated per head,
 *         pair (2i, 2i+1) by angle pos * theta^(-2i/head_dim); V untouched.
 *   [PFD] "SwiGLU: a gate in the FFN, paid for with a narrower hidden
 *         layer": hidden = 2/3 * 4d rounded up to a multiple of 256.
 *   [NAR] "GQA Was Not an Original LLaMA Feature": the KV cache read by
 *         autoregressive decoding.
 *
 * Conventions for every entry point below
 *   - Pointers named d_* are DEVICE pointers; h_* are HOST pointers.  The
 *     caller owns every buffer it passes and keeps it alive until the work
 *     queued on `stream` has finished.  The model lives in one
 *     caller-allocated device arena and the single ops work on caller
 *     buffers: no entry point allocates device memory, except the
 *     failure-detection self-test llama_debug_gemm_timeout, which allocates
 *     and frees its own 80 KB operands.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on it unless stated otherwise; outputs are valid once the
 *     stream has been synchronised.
 *   - Return value: LLAMA_OK (0) or a negative llama_status.  Arguments are
 *     validated on the host before anything is queued; an invalid call
 *     queues nothing.  A failed CUDA launch returns LLAMA_ERR_CUDA.
 *   - Row-major layouts.  Weights are stored "K-major": a matrix the pages
 *     apply as x @ W with W of shape (d_in, d_out) is stored as (d_out, d_in).
 *   - Not thread-safe per model handle: one host thread drives one model.
 */
#ifndef LLAMA_B200_H
#define LLAMA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LLAMA_API __attribute__((visibility("default")))
#else
#define LLAMA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum llama_status {
    LLAMA_OK = 0,
    LLAMA_ERR_INVALID_ARG = -1, /* shape or argument outside what is supported */
    LLAMA_ERR_OOM = -2,         /* arena / workspace smaller than required */
    LLAMA_ERR_CUDA = -3,        /* a CUDA runtime call or launch failed */
    LLAMA_ERR_TIMEOUT = -4,     /* a bounded device-side wait expired */
    LLAMA_ERR_STATE = -5        /* call out of order (decode before prefill, cache full) */
} llama_status;

typedef enum llama_dtype {
    LLAMA_F32 = 0,  /* weights and activations fp32, SIMT fp32 GEMMs */
    LLAMA_BF16 = 1  /* weights and GEMM operands bf16, fp32 accumulate and trunk */
} llama_dtype;

typedef struct llama_config {
    int32_t n_layers;
    int32_t d_model;
    int32_t n_heads;
    int32_t head_dim;    /* d_model == n_heads * head_dim; head_dim in {32, 64, 128} */
    int32_t ffn_hidden;  /* 0 => 256 * ceil(floor(8 d / 3) / 256) */
    int32_t vocab;
    float norm_eps;      /* RMSNorm eps (1e-6 in every workload) */
    float rope_theta;    /* RoPE base (10000) */
    int32_t dtype;       /* llama_dtype */
    int32_t max_batch;   /* largest B passed to prefill / decode */
    int32_t max_seq;     /* prompt length + decode steps, per sequence */
    int32_t n_kv_heads;  /* key/value heads (grouped keys and values); 0 => n_heads.
                            n_heads % n_kv_heads == 0; query head h uses key/value
                            head h / (n_heads / n_kv_heads) */
    int32_t bias;        /* 1: the bias variant -- every linear layer adds a bias of its
                            output width, each in-layer RMSNorm adds a shift after the
                            gain (none on the final norm and head); fp32, drawn like
                            the weights from tensor ids 2^20 + 16 l + k */
    int32_t tp_size;     /* tensor parallelism: 0 or 1 = off; T > 1 = this model is one of
                            T shards (see llama_set_allreduce).  n_heads, n_kv_heads and
                            ffn_hidden / 128 must divide by T. */
    int32_t tp_rank;     /* this shard, 0 <= tp_rank < T */
    int32_t kv_pages;    /* 0: contiguous KV cache [L][2][max_batch][n_kv][max_seq][head_dim];
                            P > 0 (bf16 only): a pool of P pages of 128 positions,
                            [L][2][P][n_kv][128][head_dim], mapped per sequence by a page
                            table (llama_set_pages) */
} llama_config;

typedef struct llama_model llama_model; /* opaque host handle */

/* ------------------------------------------------------------------ model */

/* Device bytes the model arena must hold for `cfg`: weights ([PFD] "6.7B
 * parameters, 1T tokens: the arithmetic" counts them), RoPE table,
 * KV cache [L][2][max_batch][n_kv_heads][max_seq][head_dim], activations and
 * workspace.  Host-only; queues nothing. */
LLAMA_API int llama_model_bytes(const llama_config* cfg, uint64_t* bytes_out);

/* [PFD] "6.7B parameters, 1T tokens: the arithmetic" fixes the shapes; the
 * pages give no initialisation (their models are trained), so the weights
 * are a synthetic stand-in drawn the same way on the GPU and in the oracle.
 * Carve the model out of `d_arena` (>= llama_model_bytes, 256-byte aligned)
 * and fill the weights on the device from the counter-based generator
 * (Philox4x32-10 keyed by (seed, tensor id), Box-Muller, N(0, 0.02^2),
 * rounded to nearest-even into the storage type; RMSNorm gains 1).  Builds
 * the RoPE cos/sin table on the host in fp64 and copies it.  Synchronises
 * `stream` before returning.  *out receives a host handle freed by
 * llama_free; the arena stays owned by the caller. */
LLAMA_API int llama_init_weights(const llama_config* cfg, uint32_t seed, void* d_arena,
                       uint64_t arena_bytes, void* stream, llama_model** out);

/* [PFD] "The one formula": embedding, L pre-norm blocks, final RMSNorm and
 * head, with the causal mask of "LLaMA is a pull request against the 2017
 * transformer".
 * Causal prefill of B sequences of S tokens each (B <= max_batch,
 * 1 <= S <= max_seq).  d_tokens: int32 [B*S], row b*S + s.  Resets the KV
 * cache and sets the decode position to S.  d_logits: fp32 [B*S, vocab]
 * logits of every position, or NULL to skip the final norm and head. */
LLAMA_API int llama_prefill(llama_model* m, const int32_t* d_tokens, int32_t B, int32_t S,
                  float* d_logits, void* stream);

/* [PFD] "The one formula", causal: each sequence on its own (the pages do
 * not discuss batching; positions restart at 0 in every sequence).
 * Ragged batch: the same [B, S] token block, but sequence b holds only its
 * first h_lens[b] tokens (host int32 [B], 1 <= h_lens[b] <= S); the
 * remaining tokens are padding and must be valid ids (their rows are
 * computed and ignored: causal attention keeps them out of every valid
 * row, and decoding overwrites their cache entries).  Sequence b continues
 * at position h_lens[b]; with d_logits the greedy choice is taken at its
 * row h_lens[b] - 1.  Rows of padding positions in d_logits are
 * unspecified.  Copies h_lens to the device on `stream`. */
LLAMA_API int llama_prefill_ragged(llama_model* m, const int32_t* d_tokens, int32_t B, int32_t S,
                                   const int32_t* h_lens, float* d_logits, void* stream);

/* [PFD] "The one formula" and "Pre-norm: the norm goes on the branch, not
 * the trunk": h = x + Attn(RMSNorm(x)), y = h + FFN(RMSNorm(h)), per block.
 * The blocks alone, on a given fp32 trunk: d_x [B*S, d_model] in,
 * d_y [B*S, d_model] out (the trunk after the last block, before the final
 * norm).  Positions 0..S-1 per sequence.  d_x and d_y may alias. */
LLAMA_API int llama_prefill_trunk(llama_model* m, const float* d_x, int32_t B, int32_t S,
                        float* d_y, void* stream);

/* [NAR] "GQA Was Not an Original LLaMA Feature": autoregressive decoding
 * appends the new token's key and value to the cache and attends over all
 * cached positions.
 * One greedy decoding step for the B sequences of the last prefill: token
 * d_tokens[b] (int32 [B]) sits at its sequence's current position p_b; its
 * K and V are appended at p_b; attention spans 0..p_b.  d_next (int32 [B],
 * may be NULL): argmax of the logits, lowest id on ties.  d_logits: fp32
 * [B, vocab] or NULL.  Advances every p_b by one.  LLAMA_ERR_STATE before a
 * prefill or when the largest p_b == max_seq. */
LLAMA_API int llama_decode_step(llama_model* m, const int32_t* d_tokens, int32_t* d_next,
                      float* d_logits, void* stream);

/* [NAR] "GQA Was Not an Original LLaMA Feature": autoregressive decoding,
 * one token per step; greedy (argmax, lowest id on ties) because the pages
 * name no decoding strategy.
 * n_steps greedy steps fed back on the device: step 0 consumes
 * d_first [B] (or, when d_first is NULL, the greedy choice at the last
 * position of the preceding llama_prefill that produced logits, or the
 * token the preceding step chose); step i consumes the token step i-1
 * chose.  d_out: int32 [n_steps, B].  Replays one captured CUDA graph per
 * step (launched eagerly while profiling is enabled). */
LLAMA_API int llama_generate(llama_model* m, const int32_t* d_first, int32_t n_steps,
                   int32_t* d_out, void* stream);

/* No passage (bookkeeping of the decode positions of llama_decode_step).
 * Current decode position: the largest over the sequences (tokens held
 * per sequence in the KV cache; all equal unless the batch is ragged). */
LLAMA_API int llama_position(const llama_model* m);

/* No passage (bookkeeping).  Each sequence's position into h_out (host
 * int32, n >= B); returns B. */
LLAMA_API int llama_positions(const llama_model* m, int32_t* h_out, int32_t n);

/* No passage (bookkeeping: re-run decoding from an earlier position).
 * Move every sequence's position back to `position` (1 <= position <= the
 * smallest current position): cache entries below it are kept, later ones
 * are overwritten by the next steps.  Queued on `stream`. */
LLAMA_API int llama_rewind(llama_model* m, int32_t position, void* stream);

/* [PFD] "The one formula" (prefill) then [NAR] "GQA Was Not an Original
 * LLaMA Feature" (decoding), as llama_prefill and llama_generate.
 * End to end from HOST buffers: copy h_tokens (int32 [B*S], host; pinned
 * memory makes the copy asynchronous) to the device, prefill (logits of
 * every position into d_logits [B*S, vocab] when it is not NULL, else the
 * head runs on each sequence's last position only), then n_steps greedy
 * steps, and copy the generated tokens to h_out (int32 [n_steps, B],
 * host).  Asynchronous on `stream`: h_out is valid after a synchronise. */
LLAMA_API int llama_complete(llama_model* m, const int32_t* h_tokens, int32_t B, int32_t S,
                             float* d_logits, int32_t n_steps, int32_t* h_out, void* stream);

/* No passage (inspection).
 * Device pointer and byte size of an internal buffer, for inspection:
 * name in {"kv" (the whole cache), "trunk", "q", "attn", "act", "xn",
 * "embed", "head", "wqkv", "wo", "wgu", "wd"}; `layer` selects the layer for
 * per-layer weights.  Layouts are those of the arena described above. */
LLAMA_API int llama_model_tensor(const llama_model* m, const char* name, int32_t layer,
                       void** d_ptr, uint64_t* bytes);

/* [NAR] "GQA Was Not an Original LLaMA Feature": decoding keeps the keys and
 * values of every earlier position, per sequence.  With a paged cache
 * (kv_pages > 0) they live in pages of 128 positions taken from one pool, so
 * that sequences of different lengths need not each reserve max_seq
 * positions.  h_table (host int32 [B][pages_per_seq]) gives sequence b's
 * logical page p (positions 128 p .. 128 p + 127) as a pool page in
 * [0, kv_pages); no page may appear twice.  Positions of each sequence are
 * then limited to 128 * pages_per_seq (and max_seq).  Copies the table to
 * the device on `stream` and synchronises it.  At init, when kv_pages >=
 * max_batch * ceil(max_seq / 128), sequence b gets pages b * ceil(max_seq /
 * 128) + p; otherwise the table must be set before the first prefill
 * (LLAMA_ERR_STATE).  The pool starts zeroed. */
LLAMA_API int llama_set_pages(llama_model* m, const int32_t* h_table, int32_t B, int32_t pages_per_seq,
                              void* stream);

/* ------------------------------------------------------- tensor parallel
 * [KN] "LLaMA: Open and Efficient Foundation Language Models" knowledge
 * note, "Efficient Training Implementation": the model is split across GPUs
 * (model parallelism) and the all-reduce is hidden behind computation.
 *
 * Shard r of T holds query heads [r H/T, (r+1) H/T) and key/value heads
 * [r Hkv/T, (r+1) Hkv/T) -- their columns of Wq, Wk, Wv, their rows of Wo
 * (the attention features they produce) and their KV cache -- and FFN
 * hidden units [r h/T, (r+1) h/T): their columns of Wgate and Wup and rows
 * of Wdown.  Embedding, norms, head and the fp32 trunk are replicated.  The
 * weights a shard holds are exactly the slices of the full model's (same
 * generator, same element indices).  In each block the O and down
 * projections of a shard produce a partial sum of the full product; shard 0
 * adds its partial (and the bias variant's output bias) to the trunk, the
 * others write theirs in its place, and one all-reduce (sum) over the
 * shards then leaves the new trunk on every shard:
 *     x' = x + sum_r attn_r Wo_r,    y = x' + sum_r act_r Wdown_r.
 * Prefill (llama_prefill, llama_prefill_ragged, llama_prefill_trunk) runs
 * this way; decoding is not sharded (the decode entry points return
 * LLAMA_ERR_INVALID_ARG on a shard). */

/* Sum all-reduce of `count` floats at d_buf across the T shards, in place,
 * queued on `stream` (a cudaStream_t): every shard's d_buf must hold the
 * element-wise sum once the work queued on `stream` completes, identical on
 * every shard.  Return 0, or non-zero to abort the calling entry point with
 * LLAMA_ERR_CUDA.  Called from the host thread that made the entry-point
 * call, once per row chunk and exchange point (2 per block). */
typedef int (*llama_allreduce_fn)(float* d_buf, uint64_t count, void* stream, void* ctx);

/* [KN] "Efficient Training Implementation" (above): the all-reduce hidden
 * behind computation.
 * Installs the exchange of a shard (tp_size > 1): `fn` with `ctx` is called
 * for each all-reduce.  `chunks` (1..16) splits the token rows of every
 * projection after attention into that many blocks (multiples of 128 rows):
 * the all-reduce of block c, queued on a stream of the model's own, runs
 * while the projections of block c + 1 compute, and the next sublayer's
 * norm and projection of block c start as soon as block c's all-reduce is
 * done.  Host-only. */
LLAMA_API int llama_set_allreduce(llama_model* m, llama_allreduce_fn fn, void* ctx, int32_t chunks);

/* [KN] "Efficient Training Implementation" (above): the model split
 * across GPUs.
 * The slices shard cfg->tp_rank of cfg->tp_size holds, into h_out (host
 * int32 [6]): first query head, query heads, first key/value head,
 * key/value heads, first FFN hidden unit, FFN hidden units.  Host-only. */
LLAMA_API int llama_tp_shard(const llama_config* cfg, int32_t* h_out);

/* No passage (failure detection).
 * Reads (synchronously) and clears the sticky device error word that
 * bounded device waits set; returns LLAMA_OK or LLAMA_ERR_TIMEOUT. */
LLAMA_API int llama_last_error(llama_model* m);

/* No passage (lifetime).
 * Releases the host handle (and its captured graphs).  The arena is the
 * caller's to free afterwards. */
LLAMA_API void llama_free(llama_model* m);

/* No passage.  Static text naming a llama_status value; never NULL. */
LLAMA_API const char* llama_status_str(int status);

/* --------------------------------------------------------- instrumentation
 * No passage: measurement of the computation above, not a step of it. */

/* No passage (instrumentation).
 * Kernel launches this library has issued in this process; a replay of the
 * captured decode graph counts every kernel in it. */
LLAMA_API int64_t llama_kernel_launches(void);

/* No passage (instrumentation).
 * Per-region device timing (process-wide, host-side state).  While enabled,
 * every region of the launch sequence (one GEMM, its reduction, a norm,
 * an attention pass ...) is bracketed by CUDA events on its stream and the
 * decode step runs eagerly instead of as a graph.  Entries accumulate the
 * region's device milliseconds, kernel launches, calls, and the algorithmic
 * bytes and FLOPs of the work it was handed.  llama_profile_count()
 * synchronises on the pending events. */
LLAMA_API int llama_profile_enable(int32_t on);
LLAMA_API void llama_profile_reset(void);
LLAMA_API int llama_profile_count(void);
LLAMA_API int llama_profile_entry(int32_t i, const char** name, double* ms, int64_t* launches,
                                  int64_t* calls, double* bytes, double* flops);

/* No passage (instrumentation).
 * Phase timestamps of the last bf16 decode step run while profiling was
 * enabled: h_out (host) receives ctas * phases * 2 %globaltimer values
 * (ns), [cta][phase][start, end]; phases run embed, then per layer QKV,
 * attention, O, gate/up, down, then head and greedy choice.  With
 * h_out == NULL only *ctas and *phases are filled.  Synchronous. */
LLAMA_API int llama_step_timeline(llama_model* m, uint64_t* h_out, int64_t n, int32_t* ctas,
                                  int32_t* phases);

/* No passage (failure detection).
 * Failure-detection self-test (synchronous): runs one small tensor-core
 * GEMM whose activation tile is never requested, so the kernel's bounded
 * wait for it expires (about 2 s); the kernel records the timeout, frees
 * its tensor memory and exits.  Returns LLAMA_ERR_TIMEOUT when the
 * mechanism works (the CUDA context stays usable).  Allocates and frees its
 * own 80 KB with cudaMallocAsync. */
LLAMA_API int llama_debug_gemm_timeout(void* stream);

/* ------------------------------------------------------------ single ops
 * The kernels the model runs, exposed one by one on caller buffers.  dtype
 * selects fp32 or bf16 storage of the T-typed operands. */

/* No passage (failure detection).
 * Standalone-op error word: the single ops below (and
 * llama_op_attention_decode_noalloc) record an expired bounded device wait
 * in one word per device, as the model does in its own.  This waits for all
 * work queued on the current device (cudaDeviceSynchronize), then reads and
 * clears that device's word: LLAMA_OK, or LLAMA_ERR_TIMEOUT when a call's
 * result is incomplete (a decode-attention chunk whose keys never arrived
 * is left out of its row's softmax). */
LLAMA_API int llama_op_last_error(void);

/* y[r, :] = x[r, :] / sqrt(mean(x[r, :]^2) + eps) * g, r < rows.
 * x fp32 [rows, d]; g fp32 [d]; y dtype-typed [rows, d]; d % 4 == 0,
 * d <= 8192.  [PFD] "RMSNorm: LayerNorm minus the mean". */
LLAMA_API int llama_op_rmsnorm(int32_t dtype, const float* d_x, const float* d_g, void* d_y,
                     int32_t rows, int32_t d, float eps, void* stream);

/* [PFD] "The code": every projection is x @ W; here W is stored (d_out,
 * d_in), so the product is A W^T.
 * C = A W^T, or C += A W^T when accumulate != 0.  A dtype-typed [M, K],
 * W dtype-typed [N, K] (K-major), C fp32 [M, N].  bf16: tcgen05 tensor-core
 * GEMM, K % 64 == 0, N % 16 == 0, pointers 16-byte aligned; fp32: SIMT. */
LLAMA_API int llama_op_gemm(int32_t dtype, const void* d_A, const void* d_W, float* d_C,
                  int32_t M, int32_t N, int32_t K, int32_t accumulate, void* stream);

/* [PFD] "LLaMA is a pull request against the 2017 transformer" (attention
 * untouched, causal mask); "RoPE: rotate Q and K, leave V alone" (q and k
 * arrive rotated).
 * Causal attention, heads independent.  q, k, v dtype-typed with layout
 * [B][H][*][head_dim]; q has S rows per head, k/v have kv_stride rows per
 * head (>= S; the first S are used).  o dtype-typed [B*S, H*head_dim]:
 * row b*S + t, columns of head h at [h*head_dim, (h+1)*head_dim).
 * Scale 1/sqrt(head_dim); key j is visible to query t iff j <= t.
 * The bf16 kernel's CTAs take work items from a counter that each call
 * leaves zero: calls on one device run one at a time (stream-ordered). */
LLAMA_API int llama_op_attention_prefill(int32_t dtype, const void* d_q, const void* d_k,
                               const void* d_v, void* d_o, int32_t B, int32_t H,
                               int32_t S, int32_t head_dim, int32_t kv_stride,
                               void* stream);

/* [NAR] "GQA Was Not an Original LLaMA Feature": the decoding query reads
 * the keys and values of every earlier position.
 * Decode attention: one query per (b, h) against keys/values 0..len-1.
 * q dtype-typed [B, H*head_dim]; k, v [B][H][kv_stride][head_dim];
 * o dtype-typed [B, H*head_dim].  Split over the sequence into chunks of 128
 * keys whose partial results go to d_work (llama_op_attention_decode_work_bytes
 * bytes: fp32 partials, then int arrival counters the call clears first);
 * the last chunk of each (b, h) to finish merges them. */
LLAMA_API int llama_op_attention_decode(int32_t dtype, const void* d_q, const void* d_k,
                              const void* d_v, void* d_o, int32_t B, int32_t H,
                              int32_t len, int32_t head_dim, int32_t kv_stride,
                              void* d_work, uint64_t work_bytes, void* stream);
/* [NAR] "GQA Was Not an Original LLaMA Feature" (workspace of the decode
 * attention above): bytes of d_work llama_op_attention_decode needs for
 * B x H queries over up to max_len keys (host-only; 0 for invalid arguments). */
LLAMA_API uint64_t llama_op_attention_decode_work_bytes(int32_t B, int32_t H, int32_t max_len,
                                              int32_t head_dim);

/* [NAR] "GQA Was Not an Original LLaMA Feature", as llama_op_attention_decode.
 * The same decode attention for callers that cannot allocate device
 * memory when they call it (runtimes that plan all device memory up front,
 * code being captured into a CUDA graph that must not allocate, embedders
 * without a device allocator).  The pages have no counterpart: this is an
 * integration variant.  The split-sequence workspace is a fixed 8 MiB array
 * in the library's own device memory, held on every GPU that loads the
 * library until the process exits; this call allocates nothing.
 *   - llama_op_attention_decode_work_bytes(B, H, len, head_dim) =
 *     4 * B * H * ceil(len / 128) * (head_dim + 2) (rounded up to 16) +
 *     4 * B * H must be <= 8 MiB; larger calls return LLAMA_ERR_OOM and
 *     queue nothing.  head_dim in {32, 64, 128}.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first
 *     call before any stream capture.
 *   - All calls share the array: calls that overlap on the GPU (different
 *     streams or host threads) race.  Each call clears the array's
 *     arrival counters (a memset on `stream`) before its kernel; every
 *     other slot it reads it writes first.
 * Arguments and layouts as llama_op_attention_decode. */
LLAMA_API int llama_op_attention_decode_noalloc(int32_t dtype, const void* d_q, const void* d_k,
                                                const void* d_v, void* d_o, int32_t B, int32_t H,
                                                int32_t len, int32_t head_dim, int32_t kv_stride,
                                                void* stream);

/* Greedy choice over the (n, vocab) logits of [PFD] "The one formula".
 * out[r] = argmax_j logits[r, j] (lowest j on ties), r < rows. */
LLAMA_API int llama_op_argmax(const float* d_logits, int32_t rows, int32_t n, int32_t* d_out,
                    void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LLAMA_B200_H */
