/*
 * llama3.h -- C ABI of the B200 (sm_100a) Llama-3 decoder forward pass.
 *
 * The library computes the decoder described by the Llama-3 pages:
 *   RMSNorm -> Wq/Wk/Wv -> RoPE (pairwise complex rotation, theta = rope_theta)
 *   -> causal grouped-query attention -> wo + residual -> RMSNorm
 *   -> SwiGLU FFN w2(silu(w1 x) * w3 x) + residual,
 * and after the last block: final RMSNorm -> output projection -> argmax.
 *
 * Sources (cited by page title and section):
 *   [S1] "从0开发大模型—译llama3-from-scratch" (sunaigc.com) §2-§12
 *   [S2] "Build your own Llama 3 from scratch" (gitcode.csdn.net) §1.2 ModelArgs,
 *        §3.1 RMSNorm, §3.2 RoPE, §3.3 KV Cache, §3.4 GQA, §3.5 FeedForward,
 *        §3.6 TransformerBlock, 四 output block, 六 inference
 *   [S3] "llama3-from-scratch：输出层与预测" (agent.csdn.net) "预测流程的完整实现",
 *        "性能优化考虑"
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor arguments are DEVICE pointers into memory the caller allocated
 *    and owns (weights, activations, caches, RoPE table, workspace).  The
 *    library never allocates or frees device memory and keeps no pointer
 *    after a call returns.
 *  - Row-major, densely packed.  Linear weights are [out, in] and a Linear
 *    computes y = x W^T ([S1] §6.5, [S2] §3.4 nn.Linear(bias=False)).
 *  - Element type of activations, weights and caches is cfg->dtype:
 *    LLAMA3_DTYPE_BF16 (bfloat16, the fast tcgen05 path for head_dim >= 64;
 *    head_dim 16 and 32 run on the SIMT kernels) or LLAMA3_DTYPE_F32 (float,
 *    SIMT kernels, meant for small models).  Accumulation is fp32.
 *  - Every device pointer must be 16-byte aligned (LLAMA3_ERR_ALIGN).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and may be captured in a CUDA graph.
 *  - Return value: LLAMA3_OK (0) or an LLAMA3_ERR_* code.  Invalid arguments
 *    are rejected on the host before anything is launched.  A device-side
 *    problem (token id out of range, a bounded wait that gave up) does not
 *    trap: it is recorded in a per-device status word that
 *    llama3_device_status() reads and clears.
 */
#ifndef LLAMA3_H
#define LLAMA3_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* llama3_stream_t; /* identical to cudaStream_t */

enum llama3_dtype { LLAMA3_DTYPE_BF16 = 0, LLAMA3_DTYPE_F32 = 1 };

enum llama3_status {
  LLAMA3_OK = 0,
  LLAMA3_ERR_ARG = 1,         /* inconsistent config or size argument          */
  LLAMA3_ERR_ALIGN = 2,       /* pointer not 16-byte aligned / bad stride      */
  LLAMA3_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required    */
  LLAMA3_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed             */
  LLAMA3_ERR_TIMEOUT = 5,     /* device: a bounded wait gave up                */
  LLAMA3_ERR_TOKEN = 6,       /* device: token id outside [0, vocab)           */
  LLAMA3_ERR_UNSUPPORTED = 7  /* valid model, but no kernel for this shape     */
};

/*
 * Model hyper-parameters -- the ModelArgs / params.json fields of [S1] §2 and
 * [S2] §1.2.  Constraints checked by every call:
 *   dim == n_heads * head_dim; n_heads % n_kv_heads == 0; head_dim even and
 *   in {16, 32, 64, 96, 128}; ffn_hidden >= 1;
 *   norm_eps > 0; rope_theta > 1; dim and ffn_hidden multiples of 8 for bf16,
 *   of 4 for fp32.
 * ffn_hidden is taken as given (the caller applies the hidden-size rule of
 * [S2] §3.5 if it wants it).  vocab is only needed by the LM head / embedding.
 */
typedef struct llama3_config {
  int dim;         /* model width D                                   */
  int n_heads;     /* query heads H                                   */
  int n_kv_heads;  /* key/value heads KV (query head h uses h/(H/KV)) */
  int head_dim;    /* hd = D / H                                      */
  int ffn_hidden;  /* F                                               */
  int vocab;       /* V (0 if no embedding / LM head is used)         */
  float norm_eps;  /* RMSNorm epsilon                                 */
  double rope_theta;
  int dtype;       /* enum llama3_dtype                               */
} llama3_config;

/*
 * Weights of one decoder block, checkpoint names of [S1] §2.  All [out, in]:
 *   attention_norm, ffn_norm : [D]
 *   wqkv : [(H + 2*KV) * hd, D]  -- the rows of wq, wk, wv stacked in that
 *          order (torch.cat((wq, wk, wv), 0)); head j of q is rows j*hd..
 *   wo   : [D, H*hd]
 *   w1, w3 : [F, D]    (gate and value paths of SwiGLU, [S2] §3.5)
 *   w2   : [D, F]
 */
typedef struct llama3_layer_weights {
  const void* attention_norm;
  const void* wqkv;
  const void* wo;
  const void* ffn_norm;
  const void* w1;
  const void* w2;
  const void* w3;
} llama3_layer_weights;

/*
 * RoPE table ([S1] §6.7, [S2] §3.2 precompute_freqs_cis).
 * Writes cos_sin[m][i][0] = cos(m * theta_i), cos_sin[m][i][1] = sin(m * theta_i)
 * with theta_i = theta^(-2i/head_dim), i < head_dim/2, 0 <= m < max_pos.
 * Angles are evaluated in double precision on the host and stored as float;
 * the table (max_pos * head_dim * 4 bytes, device memory) is copied with one
 * cudaMemcpyAsync on `stream`.  The pages build 2*max_seq_len positions.
 * Errors: LLAMA3_ERR_ARG (head_dim odd or < 2, max_pos < 1, theta <= 1).
 */
int llama3_init_rope_table(float* cos_sin, int head_dim, int max_pos, double theta,
                           llama3_stream_t stream);

/*
 * Bytes of workspace that llama3_layer_forward (seq tokens per sequence),
 * llama3_layer_decode and llama3_lm_head_argmax (up to lm_rows rows) need
 * for this config and batch.  One buffer of that size serves all three.
 */
int llama3_workspace_size(const llama3_config* cfg, int batch, int seq, int lm_rows,
                          size_t* bytes);

/*
 * Token embedding gather x[t] = table[ids[t]] ([S1] §4, [S2] 四 tok_embeddings).
 * ids: int32 [n_tokens]; table: [vocab, D]; x: [n_tokens, D].  An id outside
 * [0, vocab) writes a zero row and records LLAMA3_ERR_TOKEN on the device.
 */
int llama3_embed(const llama3_config* cfg, const int32_t* ids, const void* table, void* x,
                 int n_tokens, llama3_stream_t stream);

/*
 * Prefill / chunked prefill of one decoder block ([S2] §3.6 TransformerBlock,
 * §3.4 Attention.forward with start_pos), in place:
 *   x <- h + FFN(RMSNorm(h)),  h = x + Attn(RMSNorm(x))
 * x: [batch, seq, D] (in/out).  k_cache, v_cache: [batch, cache_cap, KV, hd];
 * this call writes the rotated keys and the values of positions
 * [start_pos, start_pos + seq) and attends, for the token at position
 * p = start_pos + t, to cached positions 0..p (causal, diagonal included).
 * rope: table from llama3_init_rope_table with rope_len >= start_pos + seq.
 * ws: workspace of at least llama3_workspace_size(cfg, batch, seq, .) bytes.
 * Errors: LLAMA3_ERR_ARG (start_pos + seq > cache_cap, batch/seq < 1, ...),
 * LLAMA3_ERR_ALIGN, LLAMA3_ERR_WORKSPACE, LLAMA3_ERR_CUDA.
 */
int llama3_layer_forward(const llama3_config* cfg, const llama3_layer_weights* w,
                         const float* rope, int rope_len, void* x, void* k_cache,
                         void* v_cache, int cache_cap, int batch, int seq, int start_pos,
                         void* ws, size_t ws_bytes, llama3_stream_t stream);

/*
 * llama3_layer_forward with the document-level attention mask of
 * "Build your own Llama 3 from scratch" 附 1: several documents packed into one
 * sequence must not attend to each other.  doc_start: device int32
 * [batch, seq]; doc_start[b][t] is the position where the document of token t
 * (position start_pos + t) begins.  The token then attends to positions
 * doc_start[b][t] .. start_pos + t.  Values must be non-decreasing in t and
 * lie in [0, start_pos + t] (larger values are clamped to start_pos + t).
 * Errors as llama3_layer_forward, plus LLAMA3_ERR_ARG for a NULL doc_start.
 */
int llama3_layer_forward_docs(const llama3_config* cfg, const llama3_layer_weights* w,
                              const float* rope, int rope_len, void* x, void* k_cache,
                              void* v_cache, int cache_cap, int batch, int seq, int start_pos,
                              const int32_t* doc_start, void* ws, size_t ws_bytes,
                              llama3_stream_t stream);

/*
 * One decode step of one block ([S2] 六 generate: one new token per sequence
 * against the KV cache, §3.3).  Same as llama3_layer_forward with seq = 1:
 * x: [batch, 1, D]; the new token of every sequence sits at position
 * start_pos, its k/v are written there, and it attends to positions
 * 0..start_pos.  Uses split-KV attention and split-K weight streaming.
 */
int llama3_layer_decode(const llama3_config* cfg, const llama3_layer_weights* w,
                        const float* rope, int rope_len, void* x, void* k_cache,
                        void* v_cache, int cache_cap, int batch, int start_pos, void* ws,
                        size_t ws_bytes, llama3_stream_t stream);

/*
 * One decode step of one block for a ragged batch ([S2] 六 generate with
 * sequences of different lengths; the cache of §3.3): as llama3_layer_decode,
 * but sequence b's new token sits at its own position positions[b] (device
 * memory, int32 [batch]): its k/v are written there and it attends to
 * positions 0..positions[b] of its own cache.  max_position is an upper bound
 * of every positions[b], known to the caller without reading the device
 * array (it sizes the launches; max_position + 1 <= cache_cap and <=
 * rope_len).  A position outside [0, max_position] is clamped and reported as
 * LLAMA3_ERR_ARG through llama3_device_status.  Errors as
 * llama3_layer_decode, plus LLAMA3_ERR_ARG for positions == NULL and
 * LLAMA3_ERR_ALIGN if it is not 4-byte aligned.
 */
int llama3_layer_decode_ragged(const llama3_config* cfg, const llama3_layer_weights* w,
                               const float* rope, int rope_len, void* x, void* k_cache,
                               void* v_cache, int cache_cap, int batch, const int32_t* positions,
                               int max_position, void* ws, size_t ws_bytes,
                               llama3_stream_t stream);

/*
 * One decode step of one block, as llama3_layer_decode (positions == NULL:
 * every sequence at start_pos) or llama3_layer_decode_ragged (positions !=
 * NULL, start_pos then being max_position), for a loop over the blocks that
 * hands the normalised input from one block to the next instead of
 * normalising it again ([S2] 三 TransformerBlock: the next block's first step
 * is RMSNorm of this block's output).
 *   next_attention_norm (nullable, bf16 [D], 16-byte aligned): the next
 *     block's attention-norm weight; the block's last residual step then also
 *     leaves RMSNorm(x_out, next_attention_norm) in the workspace.
 *   input_normalised: nonzero when the previous call on this workspace, for
 *     the same batch, was given this block's attention_norm as its
 *     next_attention_norm; the block then skips its first RMSNorm.  The
 *     library cannot check this: any other call on the same workspace in
 *     between (an LM head, a prefill, a decode of another batch or block)
 *     overwrites the normalised rows, and the flag then gives a wrong block
 *     output.
 * Only the tcgen05 decode path (bf16, batch <= 256 or ragged) hands the
 * normalised input on; the other paths ignore both arguments and normalise x
 * themselves, so the result is the same either way.  Errors as
 * llama3_layer_decode / llama3_layer_decode_ragged, plus LLAMA3_ERR_ALIGN for
 * a misaligned next_attention_norm.
 */
int llama3_layer_decode_chained(const llama3_config* cfg, const llama3_layer_weights* w,
                                const float* rope, int rope_len, void* x, void* k_cache,
                                void* v_cache, int cache_cap, int batch, int start_pos,
                                const int32_t* positions, const void* next_attention_norm,
                                int input_normalised, void* ws, size_t ws_bytes,
                                llama3_stream_t stream);

/*
 * One decode step through a whole block stack ([S2] 四 Transformer.forward
 * with one new token per sequence, 六 generate): block i of n_layers runs with
 * layers[i] and the caches k_caches[i], v_caches[i] (host arrays of device
 * pointers, [batch, cache_cap, KV, hd] each), in order, on x [batch, 1, D]
 * (in: the embedded tokens; out: the last block's output, before the final
 * norm).  positions == NULL: every token sits at start_pos; otherwise
 * sequence b's token at positions[b] (device int32 [batch]) and start_pos
 * bounds them all, as in llama3_layer_decode_ragged.  The same as calling
 * llama3_layer_decode_chained for i = 0 .. n_layers-1 (each block handing the
 * next its normalised input), as one call; every argument is checked for
 * every block before the first launch.
 * Errors as llama3_layer_decode for each block, plus LLAMA3_ERR_ARG for
 * n_layers < 1 or NULL arrays.
 */
int llama3_decode_step(const llama3_config* cfg, const llama3_layer_weights* layers, int n_layers,
                       const float* rope, int rope_len, void* x, void* const* k_caches,
                       void* const* v_caches, int cache_cap, int batch, int start_pos,
                       const int32_t* positions, void* ws, size_t ws_bytes, llama3_stream_t stream);

/*
 * Output block ([S1] §11-12, [S3] 预测流程): for each of `rows` hidden rows
 * h[r] = h + r*row_stride (elements), compute logits = RMSNorm(h[r], norm_w)
 * W_out^T over the vocabulary and ids_out[r] = argmax (lowest index on ties).
 * w_out: [vocab, D].  logits_out: float [rows, vocab] or NULL (not written).
 * row_stride lets a caller pick e.g. the last position of every sequence
 * without a copy (row_stride = seq*D, h = x + (seq-1)*D).
 * Errors: LLAMA3_ERR_ARG (rows < 1, vocab < 1, row_stride < D), ALIGN,
 * WORKSPACE, CUDA.
 */
int llama3_lm_head_argmax(const llama3_config* cfg, const void* norm_w, const void* w_out,
                          const void* h, int rows, long long row_stride, int32_t* ids_out,
                          float* logits_out, void* ws, size_t ws_bytes,
                          llama3_stream_t stream);

/*
 * LM head + argmax without a caller-provided workspace.
 *
 * No counterpart on the pages: this is a convenience for hosts that cannot
 * hand the library a workspace -- for example a C program embedded in a
 * server whose device memory is already carved up by another allocator, or
 * a caller that is not allowed to grow its device footprint after start-up.
 * Everything else is as llama3_lm_head_argmax: same arguments (minus ws and
 * ws_bytes), same kernels, same results.
 *
 * Scratch: the normalised rows and the per-row argmax keys live in one fixed
 * array of LLAMA3_NOALLOC_SCRATCH_BYTES (4 MiB) that the library declares as a
 * device global, so every GPU that loads the library holds those 4 MiB until
 * the process exits.  The call needs  roundup(rows * 8, 256) +
 * rows * dim * sizeof(element)  bytes of it and returns LLAMA3_ERR_WORKSPACE
 * when that exceeds the array (for dim 4096 in bf16: at most 511 rows).
 * Set-up: each call made outside a stream capture looks up the array's
 * device address (cudaGetSymbolAddress) in the current device's context, so
 * a context torn down and created again gets its own address; make the first
 * call on a device before any stream capture.  All calls share the one array
 * and find the previous call's contents there (the argmax keys are
 * re-initialised by each call): calls whose executions overlap on the GPU
 * (other streams, other host threads) race on it and must be serialised by
 * the caller.  The library allocates nothing for this call.
 */
#define LLAMA3_NOALLOC_SCRATCH_BYTES (4u << 20)
int llama3_lm_head_argmax_noalloc(const llama3_config* cfg, const void* norm_w, const void* w_out,
                                  const void* h, int rows, long long row_stride,
                                  int32_t* ids_out, float* logits_out, llama3_stream_t stream);

/*
 * Temperature / top-p draw of the next token ([S2] 六 generate and
 * sample_top_p).  For each row r of fp32 logits (row r at logits + r*ld,
 * `vocab` entries) writes ids_out[r]:
 *   temperature <= 0: the argmax (lowest index on ties), the page's T = 0 case;
 *   otherwise p = softmax(logits / temperature); tokens ranked by descending p
 *   (ties: lower index first) are kept while the probability ranked before
 *   them is <= top_p (top_p >= 1 keeps all, top_p = 0 keeps the top token);
 *   one kept token is drawn with probability proportional to p.
 * The draw is deterministic in (seed, counter, row): the first 64-bit word of
 * Philox-4x64-10 (Salmon et al., SC 2011) with key (seed, 0) and counter
 * (offset + positions[r], r, 0, 0) -- just offset when positions is NULL --
 * selects the token by the inverse CDF of the kept law taken in index order.
 * Probabilities are evaluated in fp32 and summed exactly as integers in units
 * of 2^-40 of the largest one.  Pass each sequence's current position (device
 * int32 [rows]) or the step number as offset to get a fresh draw per step.
 * Errors: LLAMA3_ERR_ARG (null pointers, rows < 1, vocab < 1, ld < vocab,
 * top_p < 0 or NaN, temperature NaN), LLAMA3_ERR_ALIGN (pointers not 4-byte
 * aligned), LLAMA3_ERR_CUDA.  Allocates nothing; asynchronous on `stream`.
 */
int llama3_sample_top_p(const float* logits, int rows, long long ld, int vocab, float temperature,
                        float top_p, unsigned long long seed, unsigned long long offset,
                        const int32_t* positions, int32_t* ids_out, llama3_stream_t stream);

/*
 * out[r] = x[row_index[r]] for r < rows: copies `dim` elements per row (x rows
 * n_rows of them, row_stride elements apart; out dense [rows, dim]).  With a
 * batch of prompts of different lengths padded to a common S, the LM head of
 * the first new token reads row b*S + len[b] - 1 of every sequence this way
 * (the padded prefill is exact on each sequence's own rows: causal attention
 * never lets a real token see a padding row).  No counterpart on the pages.
 * An index outside [0, n_rows) zeroes that row and reports LLAMA3_ERR_ARG
 * through llama3_device_status.  Errors: LLAMA3_ERR_ARG, LLAMA3_ERR_ALIGN
 * (x, out not 16-byte aligned, rows not 16-byte multiples, row_index not
 * 4-byte aligned).
 */
int llama3_gather_rows(const llama3_config* cfg, const void* x, long long row_stride, int n_rows,
                       const int32_t* row_index, int rows, void* out, llama3_stream_t stream);

/*
 * Device-side bookkeeping of one generation step, so that a whole step
 * (embed -> llama3_layer_decode_ragged per block -> LM head / draw -> this
 * call) can be captured once in a CUDA graph and replayed: every argument is
 * a device pointer whose contents change, none is a host value.
 * history[*step][b] = ids[b] for b < batch (skipped once *step >= history_rows;
 * row stride history_stride >= batch), positions[b] += 1, *step += 1.
 * End token ([S2] 六 generate stops a sequence at its end token and the loop
 * once every sequence has stopped): with eos_id >= 0, done is device int32
 * [batch + 1] (zeroed by the caller before the first step).  A sequence whose
 * done[b] is set has ids[b] replaced by eos_id before it is recorded (so it
 * keeps emitting the end token and feeds it to the next step); a sequence
 * whose ids[b] == eos_id gets done[b] = 1; done[batch] is set to 1 once every
 * sequence is done, for the host to end the loop.  eos_id < 0: done is not
 * used (may be NULL) and ids is not written.
 * Errors: LLAMA3_ERR_ARG (null pointers, done NULL with eos_id >= 0,
 * batch < 1, history_rows < 1, history_stride < batch), LLAMA3_ERR_ALIGN
 * (pointers not 4-byte aligned).
 */
int llama3_generation_advance(int32_t* positions, int32_t* ids, int32_t* history, int32_t* step,
                              int32_t* done, int eos_id, int batch, int history_rows,
                              long long history_stride, llama3_stream_t stream);

/* ---- building blocks (the steps of the calls above, exposed for tests) ---- */

/* y[r] = x[r] / sqrt(mean(x[r]^2) + eps) * w  ([S1] §5, [S2] §3.1); x rows at
 * x + r*row_stride, y dense [rows, D]. */
int llama3_rmsnorm(const llama3_config* cfg, const void* x, long long row_stride,
                   const void* w, void* y, int rows, llama3_stream_t stream);

/* y[m, n] = sum_k x[m, k] * w[n, k] (+ residual[m, n] when residual != NULL);
 * x: [m, k], w: [n, k], y/residual: [m, n] (residual may equal y).  k and n
 * multiples of 8 for bf16, n a multiple of 4 for fp32.  Uses the same GEMM
 * kernels as the layer calls. */
int llama3_linear(const llama3_config* cfg, const void* x, const void* w, const void* residual,
                  void* y, int m, int n, int k, void* ws, size_t ws_bytes,
                  llama3_stream_t stream);

/* Causal GQA attention alone ([S2] §3.4): q: [batch, seq, H, hd] (already
 * rotated), caches as in llama3_layer_forward (already holding positions
 * 0..start_pos+seq-1), out: [batch, seq, H*hd].  seq == 1 uses the decode
 * (split-KV) kernel. */
int llama3_attention(const llama3_config* cfg, const void* q, const void* k_cache,
                     const void* v_cache, int cache_cap, int batch, int seq, int start_pos,
                     void* out, void* ws, size_t ws_bytes, llama3_stream_t stream);

/* ---- measurement hooks (for benchmarks; no effect on results) ---- */

/* Kernel families a launch timer can follow. */
enum llama3_kernel_kind {
  LLAMA3_KERNEL_GEMM_QKV = 1,          /* prefill Wqkv GEMM + RoPE + cache scatter */
  LLAMA3_KERNEL_GEMM_WO = 2,           /* prefill wo GEMM + residual               */
  LLAMA3_KERNEL_GEMM_W13 = 3,          /* prefill w1|w3 GEMM + SwiGLU              */
  LLAMA3_KERNEL_GEMM_W2 = 4,           /* prefill w2 GEMM + residual               */
  LLAMA3_KERNEL_ATTENTION = 5,         /* prefill causal GQA attention             */
  LLAMA3_KERNEL_DECODE_GEMM = 6,       /* weight-streaming GEMMs (decode)          */
  LLAMA3_KERNEL_DECODE_ATTENTION = 7,  /* split-KV decode attention (main kernel)  */
  LLAMA3_KERNEL_LM_HEAD = 8,           /* LM-head GEMM + argmax                    */
  LLAMA3_KERNEL_NORM = 9,              /* RMSNorm                                  */
  LLAMA3_KERNEL_ELEMENTWISE = 10,      /* embedding, split-K reductions, misc.     */
  LLAMA3_KERNEL_SAMPLE = 11            /* temperature / top-p draw                 */
};

/* Record start_events[i] / stop_events[i] (cudaEvent_t handles created by the
 * caller) on the launching stream around each of the next n_pairs launches
 * of kernel family `kind`; n_pairs = 0 switches the timer off.  Not
 * thread-safe: meant for a single benchmarking thread. */
int llama3_set_launch_timer(int kind, void* const* start_events, void* const* stop_events, int n_pairs);

/* Number of event pairs recorded since the last llama3_set_launch_timer. */
int llama3_launch_timer_used(void);

/* Kernels launched by this library since it was loaded (all threads). */
unsigned long long llama3_launch_count(void);

/* llama3_attention with the document mask (doc_start as in
 * llama3_layer_forward_docs); always uses the prefill kernels. */
int llama3_attention_docs(const llama3_config* cfg, const void* q, const void* k_cache,
                          const void* v_cache, int cache_cap, int batch, int seq, int start_pos,
                          const int32_t* doc_start, void* out, void* ws, size_t ws_bytes,
                          llama3_stream_t stream);

/* ---- status ---- */

/* Static text for a status code. */
const char* llama3_status_string(int status);

/* Reads and clears the current device's status word (synchronises the
 * device).  *out receives LLAMA3_OK or the first device-side LLAMA3_ERR_*
 * recorded since the last call.  Returns LLAMA3_ERR_CUDA if the read fails. */
int llama3_device_status(int* out);

/* cudaError_t of the last call that returned LLAMA3_ERR_CUDA (0 if none). */
int llama3_last_cuda_error(void);

/* Kernel selection: 0 (default) = tcgen05/TMA kernels for bf16, 1 = the plain
 * SIMT kernels for every dtype (any other value selects 0).  Returns the
 * previous value. */
int llama3_set_kernel_path(int path);

/* Limit, in milliseconds, of every bounded device-side wait (default 2000). */
int llama3_set_wait_limit_ms(int ms);

/* Failure-detection test hook, off (0) by default.  Every wait of one role of
 * a kernel for another is bounded (llama3_set_wait_limit_ms): when it runs
 * out, the kernel records LLAMA3_ERR_TIMEOUT in the status word, lets its
 * copies in flight land, frees its tensor memory and returns, and the context
 * stays usable.  This hook makes such a wait run out on purpose:
 *   1: in the tcgen05 GEMMs, the first epilogue warp of every CTA leaves out
 *      its release of the accumulator after the CTA's first tile, so the MMA
 *      issuer's wait for that buffer gives up (needs three tiles per CTA);
 *   2: in the prefill attention kernel, one softmax thread of every CTA leaves
 *      out its P arrival on its first key tile, so the MMA issuer's wait for
 *      P gives up.
 * Nothing else changes; results of such a call are undefined.  Returns the
 * previous value (values other than 1 and 2 select 0). */
int llama3_set_test_withheld_arrival(int which);

/* 1 (default): kernels are launched with programmatic stream serialization,
 * so a kernel's launch and set-up overlap the end of the previous kernel in
 * the stream (each kernel waits for its predecessor before touching memory);
 * 0: ordinary launches.  Returns the previous value. */
int llama3_set_programmatic_launch(int on);

#ifdef __cplusplus
}
#endif

#endif /* LLAMA3_H */
