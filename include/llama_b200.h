/*
 * llama_b200.h - C ABI of the B200 (sm_100a) LLaMA decoder-block library.
 *
 * The library computes the forward pass of the LLaMA decoder with a KV-cache:
 * token-embedding gather, per block pre-norm RMSNorm, the fused Q/K/V
 * projection with interleaved-pair RoPE and the cache append in its epilogue,
 * causal grouped-query attention over the cache (a flash-style prefill kernel
 * for T > 1, a split-K flash-decode kernel for T == 1), the output projection
 * plus residual, the second RMSNorm, the SwiGLU FFN w2(silu(w1 x) * w3 x) plus
 * residual, and for whole-model calls the final RMSNorm and the LM head.
 *
 * Sources (pages), cited by title and section:
 *  - "LLaMA: Open and Efficient Foundation Language Models" (notes,
 *    unpurerationalist.github.io), section 3 code: ModelArgs, RMSNorm,
 *    precompute_freqs_cis, apply_rotary_emb, repeat_kv, Attention,
 *    FeedForward, TransformerBlock, Transformer.
 *  - "灵哥讲llama3(中)" (blog.csdn.net), Transformer class: rope_theta and the
 *    causal mask when the cache already holds start_pos tokens.
 *  - LLaMA model.py walk-through (linkmax.top), section 2.3 RoPE (the
 *    element-wise rotation) and section 3.2 model.
 *  - "LLaMa-1/2/3 原理+源码——拆解" (aitechtogether.com), section KV-Cache.
 *
 * Conventions for every call:
 *  - Pointers named *_dev are device pointers; the caller owns them and the
 *    library only borrows them for the duration of the call. Pointers named
 *    *_host are host pointers.
 *  - "act" is the activation/weight storage type chosen at create time:
 *    float (LLAMA_FP32) or bfloat16 (LLAMA_BF16). Accumulation is always fp32.
 *    The residual stream h is always fp32.
 *  - Calls that take a cuda_stream (a cudaStream_t, may be NULL for the
 *    legacy default stream) are asynchronous and stream-ordered; the library
 *    synchronises inside them only where it must allocate (workspace growth,
 *    first use of a private scratch) and where llama_generate releases the
 *    previous call's graph, so once llama_reserve has sized the workspace for
 *    the largest call they can be captured in a CUDA graph.
 *  - Every int-returning call returns LLAMA_OK (0) or a negative error code;
 *    an error returned before any launch leaves all state unchanged.
 *    Problems only the device can see (a token id out of range, a position
 *    past the cache, a bounded wait that timed out) set a device flag that
 *    llama_get_error reads back.
 *  - A context belongs to the device that was current at llama_create (its
 *    calls make that device current) and is used by one host thread at a
 *    time; calls on different contexts may run concurrently.
 */
#ifndef LLAMA_B200_H
#define LLAMA_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* storage types */
#define LLAMA_FP32 0
#define LLAMA_BF16 1

/* return codes */
#define LLAMA_OK 0
#define LLAMA_ERR_INVALID_ARGS -1 /* a size or shape rule below is broken */
#define LLAMA_ERR_OOM -2          /* device allocation failed */
#define LLAMA_ERR_CUDA -3         /* a CUDA runtime/driver call failed */
#define LLAMA_ERR_NOT_READY -4    /* weights for a needed layer/head not set */
#define LLAMA_ERR_TOO_LARGE -5    /* a size needs more than llama_linear_noalloc's fixed scratch */
#define LLAMA_ERR_INTERNAL -6     /* an internal consistency check failed (llama_selfcheck_plans) */
#define LLAMA_ERR_TOKEN_RANGE -10 /* device flag: a token id outside [0, vocab_size) */
#define LLAMA_ERR_POS_RANGE -11   /* device flag: start_pos[b] + s outside [0, max_seq_len) */
#define LLAMA_ERR_TIMEOUT -12     /* device flag: a bounded in-kernel wait gave up */

/* GEMM path selection for llama_linear (diagnostics) */
#define LLAMA_PATH_AUTO 0
#define LLAMA_PATH_TCGEN05 1 /* TMA + tcgen05/TMEM tensor-core GEMM (bf16) */
#define LLAMA_PATH_GEMV 2    /* weight-streaming split-K kernel for M <= 32 (bf16) */
#define LLAMA_PATH_SIMT 3    /* fp32 CUDA-core tiled GEMM (fp32 or bf16) */
#define LLAMA_WEIGHTS_TILED 16 /* OR-ed into a path: w holds llama_tile_weights tiles (bf16, GEMV or TCGEN05) */

/* Kernels of decode calls (T == 1), llama_set_decode_kernel */
#define LLAMA_DECODE_AUTO 0       /* the library's choice: currently LAYERED (measured faster) */
#define LLAMA_DECODE_LAYERED 1    /* a kernel per step: RMSNorm, GEMV, attention, GEMV, RMSNorm, GEMV, GEMV */
#define LLAMA_DECODE_PERSISTENT 2 /* always the persistent launch; an ineligible decode call fails */

/* Decode attention kernel of the per-step launches, llama_set_decode_attention */
#define LLAMA_ATTN_AUTO 0    /* the library's choice by size (see llama_set_decode_attention) */
#define LLAMA_ATTN_CHUNKED 1 /* a CTA per (sequence, kv head group, chunk of keys) */
#define LLAMA_ATTN_STREAMK 2 /* the key tiles of all sequences dealt out evenly over two CTAs per SM */

/* Product of the batched decode GEMV (9..32 tokens), llama_set_decode_linear_mma */
#define LLAMA_GEMV_MMA_AUTO 0    /* the library's choice: currently WARP (measured as fast or faster) */
#define LLAMA_GEMV_MMA_WARP 1    /* warp-level mma.sync, weights and tokens through ldmatrix */
#define LLAMA_GEMV_MMA_TCGEN05 2 /* tcgen05.mma from shared memory, accumulators in tensor memory */

/*
 * ModelArgs of the notes' section 3 code plus rope_theta ("灵哥讲llama3(中)",
 * Transformer class) and the storage type.
 *  dim, n_layers, n_heads, n_kv_heads (n_kv_heads <= 0 means n_kv_heads = n_heads),
 *  vocab_size (0 for single-block use), multiple_of, ffn_dim_multiplier
 *  (<= 0 means None), norm_eps, rope_theta, max_batch_size, max_seq_len, dtype,
 *  rope_half_split.
 * rope_half_split = 0: RoPE rotates the interleaved pairs (2i, 2i+1) of each
 *  head (the notes' apply_rotary_emb, complex form). rope_half_split = 1: the
 *  weights are given in the half-split convention of the HuggingFace port
 *  ("LLaMa-1/2/3 原理+源码——拆解", RoPE: q*cos + rotate_half(q)*sin, pairs
 *  (i, i + head_dim/2)); the library permutes the rows of wq and wk into the
 *  interleaved order at load time (dot products q.k are unchanged) and
 *  llama_kv_read/llama_kv_write present K in the half-split order.
 * Rules: dim % n_heads == 0; head_dim = dim / n_heads in {64, 128};
 *  n_heads % n_kv_heads == 0 (any ratio n_rep = n_heads / n_kv_heads, as the
 *  notes' repeat_kv allows; the attention kernels serve a kv head's n_rep query
 *  heads in groups that divide n_rep); dim % 64 == 0; all sizes positive.
 */
typedef struct {
  int32_t dim;
  int32_t n_layers;
  int32_t n_heads;
  int32_t n_kv_heads;
  int32_t vocab_size;
  int32_t multiple_of;
  float ffn_dim_multiplier;
  float norm_eps;
  float rope_theta;
  int32_t max_batch_size;
  int32_t max_seq_len;
  int32_t dtype;
  int32_t rope_half_split;
} llama_args;

typedef struct llama_ctx llama_ctx;

/*
 * The SwiGLU hidden width of the notes' FeedForward: two thirds of 4*dim
 * (truncated), times ffn_dim_multiplier when set (truncated), rounded up to a
 * multiple of multiple_of. Returns the width, or LLAMA_ERR_INVALID_ARGS.
 */
int llama_ffn_hidden(const llama_args* args);

/*
 * Create a model context on the current CUDA device: validates args,
 * allocates the packed weights, the per-layer K and V caches (zeroed, as the
 * notes' Attention.__init__ preallocates zeros), the RoPE table of
 * 2 * max_seq_len positions (precompute_freqs_cis, cos/sin in fp32) and an
 * empty workspace. *out receives the context. The library owns all of it
 * until llama_destroy.
 * Cache layout inside the library: [layer][batch][kv_head][position][head_dim]
 * (one (batch, kv head) history is contiguous); llama_kv_read/llama_kv_write
 * convert to and from the pages' [batch][position][kv_head][head_dim].
 */
int llama_create(const llama_args* args, llama_ctx** out);

/* Free everything the context owns (synchronises the device first). NULL is a no-op. */
void llama_destroy(llama_ctx* ctx);

/*
 * Copy (and pack) one block's weights from device memory in the act type,
 * nn.Linear layout [out_features][in_features], row-major:
 *  wq [n_heads*hd][dim], wk, wv [n_kv_heads*hd][dim], wo [dim][n_heads*hd],
 *  w1, w3 [ffn][dim], w2 [dim][ffn]; attn_norm, ffn_norm [dim].
 * The library packs wq|wk|wv into one matrix and interleaves the rows of w1
 * and w3 (row 2j = w1 row j, row 2j+1 = w3 row j). Synchronous with respect
 * to the host (the sources may be freed on return).
 */
int llama_set_layer(llama_ctx* ctx, int layer, const void* wq_dev, const void* wk_dev, const void* wv_dev,
                    const void* wo_dev, const void* w1_dev, const void* w2_dev, const void* w3_dev,
                    const void* attn_norm_dev, const void* ffn_norm_dev);

/*
 * Copy the token embedding [vocab][dim], the final norm weight [dim] and the
 * LM head [vocab][dim] (act type, device memory). Synchronous like llama_set_layer.
 */
int llama_set_embed_norm_head(llama_ctx* ctx, const void* tok_embeddings_dev, const void* norm_dev,
                              const void* output_dev);

/*
 * Size the workspace for calls of up to max_tokens tokens (B*T): the
 * activation buffers, and in bf16 mode, above 32 tokens, the prefill GEMM's
 * k-split scratch (256 KB per 256 x 256 output tile of the model's widest
 * linear at that many tokens, at most 3 x (SMs / 2) tiles). Calls with more tokens grow it on
 * demand, which allocates and therefore cannot be captured in a CUDA graph;
 * call this first to capture.
 */
int llama_reserve(llama_ctx* ctx, int max_tokens);

/*
 * Transformer.forward(tokens, start_pos) of the notes: tokens_dev int32 [B][T]
 * (row-major), the same start_pos for every sequence. Writes this call's keys
 * and values to cache positions start_pos .. start_pos+T-1 of sequences
 * 0..B-1 and fp32 logits to logits_dev: [B][T][vocab] when all_positions != 0,
 * else only the last position, [B][vocab].
 * Rules: 1 <= B <= max_batch_size, T >= 1, 0 <= start_pos, start_pos + T <= max_seq_len.
 */
int llama_forward(llama_ctx* ctx, const int32_t* tokens_dev, int B, int T, int start_pos, float* logits_dev,
                  int all_positions, void* cuda_stream);

/*
 * One decode step with a per-sequence position (ragged batches): tokens_dev
 * int32 [B] (T = 1), start_pos_dev int32 [B]; sequence b's new token goes to
 * cache position start_pos_dev[b] and attends to positions 0..start_pos_dev[b].
 * logits_dev fp32 [B][vocab]. A position outside [0, max_seq_len) raises
 * LLAMA_ERR_POS_RANGE on the device flag and that token's cache write is skipped.
 */
int llama_forward_ragged(llama_ctx* ctx, const int32_t* tokens_dev, const int32_t* start_pos_dev, int B,
                         float* logits_dev, void* cuda_stream);

/*
 * One TransformerBlock.forward in place on the fp32 residual stream
 * h_dev [B][T][dim]: h <- h + attn(attention_norm(h)); h <- h + ffn(ffn_norm(h)).
 * start_pos_dev int32 [B] gives each sequence's position of its first token
 * (device memory); when it is NULL, host_start_pos is used for all sequences
 * and checked on the host. Used for single-layer workloads.
 */
int llama_block_forward(llama_ctx* ctx, int layer, float* h_dev, int B, int T, const int32_t* start_pos_dev,
                        int host_start_pos, void* cuda_stream);

/*
 * Next-token selection, the LLaMA model.py walk-through (linkmax.top),
 * section 3.3 generate / sample_top_p. logits_dev fp32 [B][V] (row-major).
 * temperature <= 0: greedy, out_dev[b] = argmax_v logits[b][v] (lowest index
 * on ties). Otherwise probs = softmax(logits / temperature); sorted in
 * descending order, a token is kept when the probabilities before it sum to
 * at most top_p (0 < top_p <= 1); the kept probabilities are renormalised and
 * the token drawn is the first one, in descending order (ties in index
 * order), whose cumulative renormalised probability exceeds uniforms_dev[b]
 * (caller-supplied uniforms in [0, 1), one per sequence: the draw is
 * reproducible). out_dev int32 [B]. Uses a private, lazily allocated
 * scratch of B*V floats on the device of the first top-p call (a top-p call
 * on another device returns LLAMA_ERR_INVALID_ARGS); not thread-safe.
 * Stream-ordered.
 */
int llama_sample(const float* logits_dev, int B, int V, float temperature, float top_p, const float* uniforms_dev,
                 int32_t* out_dev, void* cuda_stream);

/*
 * generate() of the same walk-through, on the device, without host
 * round trips: tokens_dev int32 [B][total_len] holds each prompt at the
 * start of its row; prompt_mask_dev uint8 [B][total_len] is 1 where the row
 * holds a prompt token (the walk-through's input_text_mask). Starting at
 * cur = min_prompt_len (the shortest prompt), each step runs
 * Transformer.forward(tokens[:, prev:cur], prev) with last-position logits,
 * selects the next token as llama_sample does (uniforms_dev fp32
 * [total_len][B], row cur used at step cur; may be NULL when temperature <= 0)
 * and writes it to tokens[:, cur] except where the prompt mask is set; then
 * prev = cur. Cache positions 0..total_len-2 of sequences 0..B-1 are
 * overwritten. The first step (the prompt prefix) and the first decode step
 * are launched directly; the remaining decode steps replay a CUDA graph
 * captured from one step, whose column lives in device memory (plain
 * launches when there are fewer than three decode steps, or when cuda_stream
 * is itself being captured). The graph is kept until the next call or
 * llama_destroy. Rules: 1 <= B <= max_batch_size, 1 <= min_prompt_len <=
 * total_len <= max_seq_len, vocab_size > 0. Stream-ordered; tokens_dev holds
 * the result when the stream reaches the end of the call.
 */
int llama_generate(llama_ctx* ctx, int32_t* tokens_dev, const uint8_t* prompt_mask_dev, int B, int total_len,
                   int min_prompt_len, float temperature, float top_p, const float* uniforms_dev, void* cuda_stream);

/*
 * Copy one layer's caches out of / into the library, in the pages' logical
 * layout [max_batch_size][max_seq_len][n_kv_heads][head_dim], act type,
 * device memory. Stream-ordered.
 */
int llama_kv_read(llama_ctx* ctx, int layer, void* k_dev, void* v_dev, void* cuda_stream);
int llama_kv_write(llama_ctx* ctx, int layer, const void* k_dev, const void* v_dev, void* cuda_stream);

/* Zero every cache and re-arm the workspace's arrival counters (synchronous). */
int llama_reset(llama_ctx* ctx);

/*
 * Choose how decode calls (T == 1) of this context run one block
 * (LLAMA_DECODE_*). Both compute TransformerBlock.forward of the notes; they
 * differ only in the order of fp32 sums. The pages have no counterpart: this
 * is a launch-structure switch of the library.
 *  LLAMA_DECODE_LAYERED: seven kernels per block and step (RMSNorm, QKV GEMV
 *   with RoPE and the cache append, split-K decode attention, wo GEMV plus
 *   residual, RMSNorm, w1|w3 GEMV with SwiGLU, w2 GEMV plus residual).
 *  LLAMA_DECODE_PERSISTENT: one launch per block and step with one CTA per SM
 *   that streams all four weight matrices while its consumer warps walk the
 *   steps in order, separated by grid-wide barriers; the RMSNorms are fused
 *   into the loads of the linears' inputs. Eligible when dtype == LLAMA_BF16,
 *   B <= 32, head_dim == 128, dim % 128 == 0 and ffn % 64 == 0; an ineligible
 *   decode call returns LLAMA_ERR_INVALID_ARGS before any launch. The grid
 *   barriers need all of the launch's CTAs resident at once, so the kernel is
 *   a cooperative launch (no programmatic overlap with the kernel before it):
 *   a grid larger than the device can hold returns LLAMA_ERR_INVALID_ARGS
 *   before any launch, and the driver refuses the launch rather than start a
 *   grid that cannot all be resident (LLAMA_ERR_CUDA). A barrier that still
 *   waits past its bound raises LLAMA_ERR_TIMEOUT on the device flag.
 *  LLAMA_DECODE_AUTO (the default): the path measured faster on B200 for
 *   the decode workloads, currently LAYERED for every shape.
 * Returns LLAMA_ERR_INVALID_ARGS for another mode. Not stream-ordered: it
 * applies to calls made after it.
 */
int llama_set_decode_kernel(llama_ctx* ctx, int mode);

/*
 * Choose the attention kernel that decode calls (T == 1, bf16) run in the
 * per-step launches (LLAMA_ATTN_*); the persistent decode launch has its own.
 * Both compute, for every sequence b and query head h, the softmax over the
 * cached keys 0 .. start_pos[b] of kv head h / n_rep ("LLaMA: Open and
 * Efficient Foundation Language Models" notes, Attention.forward and
 * repeat_kv); they differ only in the order of fp32 sums.
 *  LLAMA_ATTN_CHUNKED: a CTA per (sequence, kv head group, chunk of up to
 *   2048 keys), merged by the CTA that finishes last.
 *  LLAMA_ATTN_STREAMK: the 64-key tiles of all (sequence, kv head group)
 *   units form one list cut into equal contiguous ranges, one per CTA, two
 *   CTAs per SM; a unit split between CTAs is merged by the last of them.
 *   Served when max_batch_size <= 1024 and head_dim is 64 or 128; a decode
 *   call of another shape returns LLAMA_ERR_INVALID_ARGS before any launch.
 *  LLAMA_ATTN_AUTO (the default): the kernel measured faster on B200 for the
 *   call's size: STREAMK when the units times the 64-key tiles of the longest
 *   history (max_seq_len for per-sequence positions) reach 8 per SM and a CTA
 *   serves at most 8 query heads (n_rep <= 8, or a multiple of 8 that is not
 *   a multiple of 16), else CHUNKED.
 * Returns LLAMA_ERR_INVALID_ARGS for another mode. Not stream-ordered: it
 * applies to calls made after it.
 */
int llama_set_decode_attention(llama_ctx* ctx, int mode);

/*
 * Choose how the decode GEMV (the weight-streaming kernel of linears with 9 to
 * 32 tokens: every decode linear of a batch of 9..32 sequences, and
 * llama_linear's LLAMA_PATH_GEMV) forms its products (LLAMA_GEMV_MMA_*). Both
 * compute y = x W^T of the notes' Attention and FeedForward linears with fp32
 * accumulation; they differ only in the order of fp32 sums within a 64-wide
 * k stage. The pages have no counterpart: this is a kernel switch of the
 * library. Process-wide (every context and llama_linear); calls of up to 8
 * tokens always take the warp-level form. Returns LLAMA_ERR_INVALID_ARGS for
 * another mode. Not stream-ordered: it applies to launches made after it.
 */
int llama_set_decode_linear_mma(int mode);

/*
 * Synchronise the device, then return and clear the device flags: LLAMA_OK,
 * or the most severe of LLAMA_ERR_TIMEOUT, LLAMA_ERR_POS_RANGE,
 * LLAMA_ERR_TOKEN_RANGE. *flags (if not NULL) receives the raw flag bits
 * (1 token range, 2 position range, 4 timeout). A pending asynchronous CUDA
 * error is returned as LLAMA_ERR_CUDA.
 */
int llama_get_error(llama_ctx* ctx, int* flags);

/*
 * Failure-detection self-test of the library's bounded device waits (the
 * pages have no counterpart). which = 0: one thread waits on an mbarrier phase
 * that nothing completes (the wait every kernel's pipeline uses); which = 1:
 * the persistent decode kernel's grid barrier, with one of its two CTAs never
 * arriving. The wait must give up after about one second, record the timeout
 * bit and return; nothing faults or traps. Synchronous (synchronises the
 * device); allocates and frees 512 bytes of device memory. *flags receives the
 * device flag bits the wait recorded (4 = timeout), *seconds the time the
 * waiting thread spent before giving up. Returns LLAMA_OK when the test ran
 * (the result is in *flags), LLAMA_ERR_INVALID_ARGS for another `which`,
 * LLAMA_ERR_CUDA or LLAMA_ERR_OOM when it could not run.
 */
int llama_selftest_bounded_wait(int which, int* flags, double* seconds);

/*
 * Host-only consistency check of the work partitions the decode kernels use
 * (the pages have no counterpart; it stands in for a sanitizer run): for M
 * tokens and a model of these sizes it walks, on the host and with the
 * kernels' own index functions, every CTA's share of the stream-K split of
 * each decode linear and of the persistent decode kernel, and checks that
 * every weight tile is covered exactly once and in bounds, that each split
 * row block's partial slots are distinct and fit the workspace, and that the
 * attention partials fit; and, for M sequences at several ragged and uniform
 * position patterns, the stream-K decode attention's split: every key tile in
 * exactly one CTA's range, each split unit merged from one partial of each CTA
 * it spans, in distinct slots inside the workspace (M up to 1024 there).
 * Returns LLAMA_OK, LLAMA_ERR_INTERNAL when a check
 * fails, or LLAMA_ERR_INVALID_ARGS for sizes the library rejects. Needs no GPU.
 */
int llama_selfcheck_plans(int M, int dim, int n_heads, int n_kv_heads, int ffn, int max_seq_len, int num_sms);

/*
 * Failure injection for out-of-memory handling (the pages have no
 * counterpart): cap the device memory the library may hold, summed over all
 * its allocations in this process (contexts, workspaces, scratch); 0 removes
 * the cap (the default). An allocation that would pass the cap fails as if the
 * device were full: the call returns LLAMA_ERR_OOM and frees what it had
 * allocated so far. llama_allocated_bytes returns the bytes the library holds
 * now (every allocation is tracked, so a failed call can be checked for
 * leaks). Thread-safe. llama_set_alloc_limit always returns LLAMA_OK.
 */
int llama_set_alloc_limit(uint64_t bytes);
uint64_t llama_allocated_bytes(void);

/* A static description of an error code. */
const char* llama_strerror(int code);

/*
 * The weight layout the library keeps for its bf16 linears (the pages have no
 * counterpart; it is a storage choice): w_dev [N][K] bf16 row-major is cut into
 * tiles of 128 rows x 64 columns, tile (n / 128, k / 64) stored contiguously
 * (16 KB) at tile index (n / 128) * (K / 64) + k / 64, rows past N zero-filled.
 * out_dev must hold ceil(N / 128) * 128 * K bf16 values. Rules: K % 64 == 0,
 * both pointers 16-byte aligned, the two regions disjoint. Stream-ordered.
 * Every decode and prefill GEMM then reads each 128 x 64 operand stage as one
 * contiguous 16 KB block.
 */
int llama_tile_weights(const void* w_dev, void* out_dev, int N, int K, void* cuda_stream);

/*
 * Diagnostics: y_dev[M][N] (fp32) = x_dev[M][K] * w_dev[N][K]^T with fp32
 * accumulation, x and w both of storage type dtype, through the chosen GEMM
 * path (LLAMA_PATH_*), optionally OR-ed with LLAMA_WEIGHTS_TILED when w_dev
 * holds llama_tile_weights tiles. Rules: M, N, K > 0, N % 8 == 0, K % 8 == 0;
 * LLAMA_PATH_GEMV needs M <= 32 and K % 64 == 0; LLAMA_PATH_TCGEN05 needs
 * dtype == LLAMA_BF16; tiled weights need dtype == LLAMA_BF16, K % 64 == 0
 * and the GEMV or TCGEN05 path. Uses a private, lazily allocated workspace
 * on the device of the first call (a call with another current device
 * returns LLAMA_ERR_INVALID_ARGS); not thread-safe.
 */
int llama_linear(const void* x_dev, const void* w_dev, float* y_dev, int M, int N, int K, int dtype, int path,
                 void* cuda_stream);

/*
 * llama_linear_noalloc: the LLAMA_PATH_GEMV case of llama_linear that
 * allocates nothing. The pages have no counterpart; this is a library
 * convenience for callers that cannot allocate device memory when they call,
 * e.g. an application whose device memory is all owned by its own pool
 * allocator, or a latency-critical loop where cudaMalloc/cudaFree (which can
 * synchronise the device) are not acceptable.
 *
 * y_dev[M][N] (fp32) = x_dev[M][K] * w_dev[N][K]^T, x and w bfloat16, fp32
 * accumulation, the same kernel as llama_linear(..., LLAMA_PATH_GEMV).
 * Rules: 1 <= M <= 32, N % 8 == 0, K % 64 == 0; the caller owns x, w, y.
 * Scratch: a fixed array of 8 MiB + 16.25 KiB of device memory compiled into
 * the library (held on every GPU where the library's device code is loaded,
 * until the process exits): at most 2 Mi fp32 split-K partial sums and 4096
 * row blocks of 128 outputs (N <= 524288). A shape that needs more returns
 * LLAMA_ERR_TOO_LARGE before anything is launched.
 * The first call on a device (with that device current) looks up the array's
 * device address; make that first call before any stream capture.
 * cudaDeviceReset unloads the array: the address looked up before it is not
 * valid afterwards, so do not call this entry point on a device after
 * resetting it (a call whose CUDA work fails forgets the address, and the
 * next call looks it up again).
 * All calls on one device share the array and it keeps the last call's
 * contents; calls whose kernels overlap on the GPU (different streams without
 * ordering between them) race. The arrival counters are cleared on
 * cuda_stream before each launch. Stream-ordered, asynchronous: the return
 * code covers only what the host can check. A bounded in-kernel wait that
 * gives up sets a bit in an error word inside the array, which stays set
 * until llama_linear_noalloc_status reads it.
 */
int llama_linear_noalloc(const void* x_dev, const void* w_dev, float* y_dev, int M, int N, int K, void* cuda_stream);

/*
 * Status of llama_linear_noalloc on the current device (the pages have no
 * counterpart): synchronises the device, copies the error word out of the
 * fixed array into a host variable, clears it, and returns LLAMA_OK or
 * LLAMA_ERR_TIMEOUT (a bounded wait of some call since the last status read
 * gave up, so that call's y is not valid); LLAMA_ERR_CUDA when the copy fails.
 * *flags (if not NULL) receives the raw bits (4 = timeout). Allocates nothing.
 */
int llama_linear_noalloc_status(int* flags);

#ifdef __cplusplus
}
#endif

#endif /* LLAMA_B200_H */
