/*
 * kie.h — C ABI of the B200 decode engine (libkie.so).
 *
 * The engine runs the autoregressive decode step of a dense decoder-only transformer
 * (pre-norm RMSNorm, rotary positions, grouped-query attention, SwiGLU MLP, untied LM
 * head, greedy argmax) as one persistent sm_100a kernel per GPU:
 *
 *  - Every weight byte and the KV cache are streamed once per generated token; decode is
 *    bound by memory bandwidth, not compute ("Kog 3000 tok/s 实时推理：内存带宽优化与请求级并发的
 *    工程权衡", section 内存带宽优化的三层策略; the HN digest of Kog's inference engine,
 *    section 技术原理).
 *  - One resident kernel replaces per-op launches (the same digest, section 技术原理;
 *    "实时AI推理为何贵56倍？持续推理与常驻内核的破局之道", section 让工作常驻 GPU). The host only
 *    writes input tokens into a mapped mailbox (the doorbell) and reads output tokens.
 *  - Sessions due on the same tick advance as one batch, so the weights are read once for
 *    the whole group (same page, section 让所有活跃会话同步推进): kie_tick.
 *  - Schedule and memory layout are fixed at kie_create, with no allocator or scheduler
 *    afterwards (same page, section 把一切提前决定好).
 *
 * Conventions for every call:
 *  - Return KIE_OK (0) or a negative kie_status. No call aborts the process.
 *  - After KIE_ERR_TIMEOUT or KIE_ERR_DEVICE the engine is poisoned: every later call
 *    except kie_last_error / kie_destroy returns KIE_ERR_STATE.
 *  - One host thread per engine; calls on one engine must not overlap.
 *  - "host" pointers are ordinary CPU memory; "device" pointers are CUDA device memory
 *    on the engine's device.
 */
#ifndef KIE_H
#define KIE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KIE_ABI_VERSION 1

typedef struct kie_engine kie_engine; /* opaque; owned by the library */
typedef int32_t kie_status;

enum {
    KIE_OK = 0,
    KIE_ERR_ARG = -1,         /* bad argument or unsupported shape                          */
    KIE_ERR_CAPACITY = -2,    /* context or session capacity exceeded; nothing was written */
    KIE_ERR_CUDA = -3,        /* a CUDA runtime call failed (message in kie_last_error)    */
    KIE_ERR_TIMEOUT = -4,     /* a host or device wait ran past timeout_ms                 */
    KIE_ERR_STATE = -5,       /* engine poisoned by an earlier timeout / device error      */
    KIE_ERR_DEVICE = -6,      /* the kernel reported an error status                       */
    KIE_ERR_UNSUPPORTED = -7  /* the engine was created without the mode this call needs  */
};

enum { KIE_FP16 = 0, KIE_BF16 = 1 };

/* Which kernels and weight layouts kie_create builds (bitmask). */
enum {
    KIE_MODE_BATCH1 = 1, /* single-session decode: kie_decode_step / kie_generate / kie_decode_launch */
    KIE_MODE_TICK = 2    /* multi-session tick and chunked prefill on tcgen05 tensor cores            */
};

typedef struct {
    int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim, ffn, vocab;
    float rms_eps;    /* RMSNorm epsilon (1e-5 in all shipped configs)                 */
    float rope_theta; /* rotary base (1e4, or 5e5 for the Llama-3-8B shape)            */
    int32_t dtype;    /* KIE_FP16 or KIE_BF16: weights and KV cache                    */
    int32_t max_sessions; /* KV slots allocated up front                               */
    int32_t max_ctx;      /* positions per session allocated up front                  */
    int32_t timeout_ms;   /* bound on every device spin and host wait of one command   */
    int32_t idle_ms;      /* the resident kernel exits after this long with no command */
    int32_t modes;        /* KIE_MODE_* bitmask                                        */
    int32_t device;       /* CUDA device ordinal                                       */
    int32_t weight_fp8;   /* 1: the batch-1 kernel streams its matrices (and the LM head) as
                             E4M3 codes with a per-row fp32 scale, quantised by kie_create
                             from the given 16-bit weights as kie_quantize_e4m3 does; half
                             the bytes per token. Needs modes == KIE_MODE_BATCH1 (the tick
                             kernel's tensor-core contractions take 16-bit operands), and
                             prompts then go through the batch-1 kernel too. 0: weights
                             stream in `dtype`.                                           */
    int32_t b1_staging;   /* where the batch-1 kernel stages streamed weights:
                             0 (default): the 3-slot shared-memory ring (64 KB slots).
                             1: the ring, plus 4 slots of tensor memory (TMEM) per SM for
                             the first 4 chunks after each layer's QKV rows, so the stream
                             runs 7 chunks ahead through the attention step; 16-bit weights
                             and d_model 2048 or 4096 only (else as 0). Same results; on
                             one B200 about as fast as 0 on the 8B shape and 4 % slower on
                             the 1.9B shape, since streaming through the attention step
                             and the grid barriers lengthens their L2 round trips.        */
    int32_t b1_kv_path;   /* how the batch-1 kernel's attention reads the KV cache:
                             0 (default): 2 when max_ctx > 8192, else 1.
                             1: plain loads from L2, the split's rows read into L2 during
                             the previous phase (best at short contexts).
                             2: bulk copies through the weight ring, 128 positions (64 KB)
                             per copy (best at long contexts, where each split's rows no
                             longer fit its read-ahead). Same results either way.          */
} kie_config;

/*
 * Weights, all DEVICE pointers in row-major [out][in] layout of the storage dtype:
 *   tok_emb [vocab][d_model], final_norm [d_model], lm_head [vocab][d_model],
 *   layers[9*l + j] for layer l, j in order: attn_norm [d], wq [Hq*D][d], wk [Hkv*D][d],
 *   wv [Hkv*D][d], wo [d][Hq*D], mlp_norm [d], w_gate [ffn][d], w_up [ffn][d], w_down [d][ffn].
 * `layers` itself is a HOST array of 9*n_layers device pointers.
 * The engine reads them only inside kie_create (it repacks them into its own arena in the
 * streaming order of its fixed schedule); the caller may free them afterwards.
 */
typedef struct {
    const void *tok_emb;
    const void *const *layers;
    const void *final_norm;
    const void *lm_head;
} kie_weights;

/* Fills a config with the shape fields zeroed and defaults for the rest
   (eps 1e-5, theta 1e4, fp16, 1 session, 4096 positions, timeouts 10 s / 200 ms,
   batch-1 mode, device 0). */
void kie_config_defaults(kie_config *cfg);

/*
 * Builds an engine: validates the shape, allocates every device buffer it will ever use
 * (packed weights, KV cache of max_sessions x max_ctx, activations, split-K scratch,
 * mapped host mailbox), computes the static work partition for this GPU's SM count and
 * repacks the weights. Constraints: d_model, n_heads*head_dim and ffn multiples of 64,
 * d_model <= 8192 (<= 4096 with KIE_MODE_BATCH1), ffn and n_heads*head_dim <= 14336;
 * head_dim one of 8, 16, 32, 64, 128; n_heads a multiple of n_kv_heads with
 * n_heads/n_kv_heads <= 8.
 * Errors: KIE_ERR_ARG (shape), KIE_ERR_CUDA (allocation or launch). On error *out is NULL.
 */
kie_status kie_create(const kie_config *cfg, const kie_weights *w, kie_engine **out);

/* Stops the resident kernel (if running) and frees everything. NULL is ignored. */
void kie_destroy(kie_engine *eng);

/* Claims a free KV slot with context length 0. KIE_ERR_CAPACITY when all are taken. */
kie_status kie_session_open(kie_engine *eng, int32_t *sid);
kie_status kie_session_close(kie_engine *eng, int32_t sid);
/* Current context length (tokens in the cache) of a session. */
kie_status kie_session_length(kie_engine *eng, int32_t sid, int32_t *ctx);
/* Rewinds a session to its first `ctx` positions (ctx <= current length); later steps overwrite the rest. */
kie_status kie_session_rewind(kie_engine *eng, int32_t sid, int32_t ctx);
/* DEVICE pointers to the session's K and V cache, each [n_layers][n_kv_heads][max_ctx][head_dim]
   of the storage dtype. Owned by the engine; valid until kie_destroy. */
kie_status kie_session_kv(kie_engine *eng, int32_t sid, void **k_dev, void **v_dev);

/*
 * Prefill, the first call of the pages' request cycle (the prompt fills the KV cache that every
 * later token reads: "Kog 3000 tok/s 实时推理…", section 内存带宽优化的三层策略).
 * Appends a prompt: tokens (HOST, n >= 1) are processed teacher-forced at positions
 * ctx..ctx+n-1, and *first_token (HOST) receives the argmax after the last one.
 * KIE_ERR_CAPACITY if ctx + n > max_ctx (nothing written). Uses the tick kernel's
 * chunked path when the engine has KIE_MODE_TICK, else the batch-1 kernel.
 */
kie_status kie_prefill(kie_engine *eng, int32_t sid, const int32_t *tokens, int32_t n, int32_t *first_token);

/*
 * One decode step (the pages' bandwidth-bound step: every weight byte and the KV cache read
 * once per token, same section) through the doorbell of the resident kernel (the host only
 * writes inputs and reads outputs: "实时AI推理为何贵56倍？…", section 让工作常驻 GPU):
 * in_token at position ctx, *out_token (HOST)
 * receives the argmax. logits_dev (DEVICE, nullable) receives the fp32 logits [vocab].
 */
kie_status kie_decode_step(kie_engine *eng, int32_t sid, int32_t in_token, int32_t *out_token, float *logits_dev);

/*
 * n greedy steps through the doorbell, the argmax fed back on the GPU with no host round
 * trip per token (the persistent single-kernel runtime of the HN digest of Kog's inference
 * engine, section 技术原理): out_tokens (HOST, [n]) receives each step's argmax.
 */
kie_status kie_generate(kie_engine *eng, int32_t sid, int32_t in_token, int32_t n, int32_t *out_tokens);

/*
 * Stream-ordered form of kie_generate: one launch of the same kernel on `stream`
 * (a cudaStream_t; NULL = the engine's own stream), reading *in_token_dev and writing
 * out_tokens_dev[n] and, if non-NULL, logits_dev[n][vocab] (all DEVICE). Returns after
 * the launch is queued; the session length advances immediately. Device errors surface
 * at the next call that synchronises (or via kie_sync).
 */
kie_status kie_decode_launch(kie_engine *eng, int32_t sid, const int32_t *in_token_dev, int32_t n,
                             int32_t *out_tokens_dev, float *logits_dev, void *stream);

/* Waits for queued launches and reports any device error they raised. */
kie_status kie_sync(kie_engine *eng);

/*
 * One tick of the continuous-inference workload ("实时AI推理为何贵56倍？…", sections
 * 让所有活跃会话同步推进 and 实测数据: all due sessions advance as one batch on a fixed
 * deadline): the n_sess sessions sids[] (HOST) advance together by `steps` greedy tokens
 * each, weights read once per step for all of them. in_tokens (HOST, [n_sess]) are the first inputs; step s's argmax is the input of
 * step s+1 on the GPU. out_tokens (HOST, [steps][n_sess]) receive every argmax.
 * logits_dev (DEVICE, nullable) receives [steps][n_sess][vocab] fp32.
 * Needs KIE_MODE_TICK; n_sess <= 64, distinct sids.
 */
kie_status kie_tick(kie_engine *eng, int32_t n_sess, const int32_t *sids, const int32_t *in_tokens, int32_t steps,
                    int32_t *out_tokens, float *logits_dev);

/*
 * Phase trace (observability). kie_trace_enable(eng, tokens) makes every later command
 * record, for its first `tokens` tokens (batch-1 decode) or steps (tick, chunked prefill), a
 * globaltimer stamp (ns) per CTA at each phase boundary; tokens = 0 turns it off. Each
 * command overwrites the record of the one before. kie_trace_read
 * copies the record into `host` (uint64, at most max_elems) and returns the element count
 * through *n; layout [cta][token][event], events per token = kie_trace_events(eng):
 * Batch-1 decode commands write one record per token:
 *   0: token start; then per layer 16 slots: 10 phase ends (0 QKV rows, 1 QKV epilogue,
 *   2 barrier, 3 attention with its slice merge, 4 O fold, 5 barrier, 6 gate/up rows,
 *   7 gate/up epilogue, 8 down fold, 9 barrier), then 10 the end of the down fold's wait for
 *   every CTA's read of the residual, 11 and 12 input vectors ready in the QKV and gate/up
 *   phases, 15 the end of this CTA's attention positions (before its split is published; 0
 *   if it had no unit); then 3 for the head (rows+argmax, barrier, final argmax); then the
 *   token's consumer ring waits in ns per weight phase (QKV rows, O fold, gate/up rows, down
 *   fold, LM head: the time thread 0 was blocked on a weight chunk that had not landed), and
 *   the producer's total wait for a free ring slot in ns.
 * Tick and chunked-prefill commands write one record per step, in the same layout:
 *   0: step start; per layer (slot 1 + 16 l + k): k = 0 first norm done, then the ends of
 *   the grid barriers after: 1 first norm, 3 QKV, 4 RoPE, 6 attention (5: this CTA's
 *   attention done, before the barrier), 7 O, 8 second norm, 9 gate/up, 10 activation,
 *   11 down; head (slot 1 + 16 L + k): 0 final norm, 1 head rows, 2 argmax.
 */
kie_status kie_trace_enable(kie_engine *eng, int32_t tokens);
kie_status kie_trace_read(kie_engine *eng, uint64_t *host, int64_t max_elems, int64_t *n);
int32_t kie_trace_events(kie_engine *eng);

/*
 * Stream-ordered form of kie_tick: one launch of the tick kernel on `stream` (cudaStream_t;
 * NULL = the engine's own stream). sids (HOST, [n_sess]) as for kie_tick; in_tokens_dev
 * (DEVICE, [n_sess]) the first inputs, out_tokens_dev (DEVICE, [steps][n_sess]) every argmax,
 * logits_dev (DEVICE, nullable, [steps][n_sess][vocab]). The last step's outputs can be passed
 * as the next call's inputs. Returns once the launch is queued; session lengths advance
 * immediately; device errors surface at kie_sync.
 */
kie_status kie_tick_launch(kie_engine *eng, int32_t n_sess, const int32_t *sids, const int32_t *in_tokens_dev,
                           int32_t steps, int32_t *out_tokens_dev, float *logits_dev, void *stream);

/*
 * Fault injection for tests of the failure paths, made on the host (no GPU fault, trap or
 * hang): with KIE_FAULT_BARRIER_SHORT the next kernel launch of this engine (resident or
 * stream-ordered, either kernel) starts its grid-barrier counter one arrival short. The
 * first grid barrier of that launch then cannot complete: every CTA's bounded wait runs out
 * after timeout_ms (the resident kernel's first barrier: idle_ms + timeout_ms), the kernel
 * records the timeout in its error word, waits for its own copies in flight, releases its
 * tensor memory and returns. The call that owns the launch reports KIE_ERR_TIMEOUT and the
 * engine is poisoned (KIE_ERR_STATE afterwards). A resident kernel is stopped first, so the
 * fault always meets a fresh launch. KIE_FAULT_NONE cancels a pending fault.
 */
enum { KIE_FAULT_NONE = 0, KIE_FAULT_BARRIER_SHORT = 1 };
kie_status kie_inject_fault(kie_engine *eng, int32_t fault);

/*
 * Sampling of one session's next tokens, the variant beside greedy argmax (used by every call
 * that produces its tokens: kie_prefill's first token, kie_decode_step, kie_generate,
 * kie_decode_launch, kie_tick, kie_tick_launch). A step's token is a function of its logits
 * and (temperature, top_k, seed, the step's position) alone:
 *   candidates: the top_k largest logits, ordered by value (descending), then index (ascending);
 *   weights:    exp((z_k - z_0) / temperature);
 *   draw:       u = (output pos + 1 of splitmix64 started from state `seed`) >> 40, / 2^24, where
 *               pos is the position of the step's input token;
 *   token:      the first candidate whose cumulative weight exceeds u * (total weight).
 * top_k = 1 is greedy argmax (temperature and seed unused). s = NULL restores greedy decoding;
 * kie_session_open starts every session greedy. Errors: KIE_ERR_ARG for top_k outside
 * [1, min(KIE_TOPK_MAX, vocab)] or, with top_k > 1, a temperature that is not a positive
 * finite number. Non-finite candidate logits fail the command with KIE_ERR_DEVICE.
 */
#define KIE_TOPK_MAX 32
typedef struct {
    float temperature;
    int32_t top_k;
    uint64_t seed;
} kie_sampling;
kie_status kie_session_sampling(kie_engine *eng, int32_t sid, const kie_sampling *s);

/*
 * Per-row E4M3 quantisation of a 16-bit matrix (w_dev: [rows][cols] of dtype, DEVICE), as
 * kie_create does for a weight_fp8 engine: scale_dev[n] (DEVICE, fp32) = max_k |w[n][k]| / 448
 * (1 for an all-zero row) and q_dev[n][k] (DEVICE, one byte each) = the E4M3 code nearest to the
 * fp32 quotient w[n][k] / scale[n] (ties to the even code), saturated at +-448. E4M3: sign, 4
 * exponent bits with bias 7, 3 fraction bits, no infinities, 0x7F / 0xFF NaN. Stream-ordered on
 * `stream` (cudaStream_t; NULL = legacy default stream). KIE_ERR_ARG on bad arguments.
 */
kie_status kie_quantize_e4m3(const void *w_dev, int64_t rows, int32_t cols, int32_t dtype, uint8_t *q_dev,
                             float *scale_dev, void *stream);

/* Copies the engine's last error message (NUL-terminated, truncated to len). */
kie_status kie_last_error(kie_engine *eng, char *buf, int32_t len);

/* Static text of a status code. */
const char *kie_status_string(kie_status s);

/*
 * Split-K single-query attention over a KV cache, as run inside the decode kernel
 * (the "attention over the KV cache" part of one decode step; see the first section
 * of this header for the passages). For query head h (kv head g = h*Hkv/Hq):
 *   out[h] = sum_{j<n_ctx} softmax_j(q[h] . K[g][j] / sqrt(D)) V[g][j].
 * q_dev [n_heads][head_dim] fp32; k_dev, v_dev [n_kv_heads][kv_stride][head_dim] of
 * dtype (kv_stride >= n_ctx positions between heads); out_dev [n_heads][head_dim] fp32;
 * scratch_dev: caller-owned DEVICE buffer of at least kie_flash_decode_scratch_bytes(...)
 * bytes (split partials and merge counters; contents on entry are ignored).
 * All DEVICE, stream-ordered on `stream` (cudaStream_t, NULL = legacy default stream).
 * n_ctx >= 1, head_dim one of 8, 16, 32, 64, 128, n_heads a multiple of n_kv_heads with
 * n_heads/n_kv_heads <= 8. Returns KIE_ERR_ARG on other shapes.
 */
kie_status kie_flash_decode(const float *q_dev, const void *k_dev, const void *v_dev, int32_t n_heads,
                            int32_t n_kv_heads, int32_t head_dim, int32_t n_ctx, int64_t kv_stride, int32_t dtype,
                            float *out_dev, void *scratch_dev, int64_t scratch_bytes, void *stream);
int64_t kie_flash_decode_scratch_bytes(int32_t n_heads, int32_t n_kv_heads, int32_t head_dim, int32_t n_ctx);

/*
 * kie_flash_decode without caller-provided scratch (the pages have no counterpart: this
 * entry point exists for callers of this library that cannot allocate device memory, such
 * as code running under a memory budget fixed at start-up, code whose device memory is
 * owned by another framework's allocator, or latency-critical loops that cannot afford the
 * device-wide stall of cudaMalloc/cudaFree).
 *
 * Same arguments and result as kie_flash_decode, minus scratch_dev/scratch_bytes. The
 * split partials and merge counters live in one static device array of
 * KIE_FLASH_DECODE_NOALLOC_MAX_BYTES, which every GPU that loads this library keeps until
 * the process exits. The call allocates nothing. The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current; make that first
 * call before any stream capture. All calls on one GPU share that GPU's array, and every
 * call leaves its partials there: calls whose kernels can overlap on the GPU (launched on
 * different streams, or from host threads without ordering between them) race with each
 * other and must be serialised by the caller; calls ordered on one stream are safe (each
 * call clears the merge counters it needs before its kernel runs).
 * The address looked up on a device's first call stays cached for the life of the process:
 * after cudaDeviceReset on that device it is stale, so a process that resets a device must
 * not call this entry point on it again. Accepted shapes are those of kie_flash_decode.
 * Returns KIE_ERR_CAPACITY when kie_flash_decode_scratch_bytes(...) for this shape exceeds
 * KIE_FLASH_DECODE_NOALLOC_MAX_BYTES, KIE_ERR_ARG for bad shapes or pointers, KIE_ERR_CUDA
 * if the address lookup or the launch fails.
 */
#define KIE_FLASH_DECODE_NOALLOC_MAX_BYTES (4 << 20)
kie_status kie_flash_decode_noalloc(const float *q_dev, const void *k_dev, const void *v_dev, int32_t n_heads,
                                    int32_t n_kv_heads, int32_t head_dim, int32_t n_ctx, int64_t kv_stride,
                                    int32_t dtype, float *out_dev, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* KIE_H */
