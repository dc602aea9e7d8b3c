// Internal definitions shared by the engine's host code and its kernels.
#pragma once
#include <stdint.h>

#include "kie.h"

#define KIE_MAX_CTAS 256
#define KIE_CONS_WARPS 16                     // consumer warps per CTA (batch-1 kernel): two groups of 8
#define KIE_CONS_THREADS (KIE_CONS_WARPS * 32)
#define KIE_THREADS (KIE_CONS_THREADS + 32)   // + one producer warp
#define KIE_NSLOT 3                           // weight ring depth
#define KIE_SLOT_BYTES 65536                  // one ring slot (large bulk copies stream best)
#define KIE_NTS 4                             // TMEM weight slots (128 columns = one 64 KB chunk each)
#define KIE_ROWACC_MAX 1024                   // output rows one CTA may own in one phase
#define KIE_GMAX 8                            // query heads per kv head
#define KIE_DMAX 128                          // head_dim
#define KIE_FOLD_MAX 256                      // inputs one CTA folds into the residual in one phase
#define KIE_B1_DMAX 4096                      // d_model the batch-1 kernel's folds support
#define KIE_KV_WARM_LINES 1024                // 128-byte lines each of K and V an attention unit reads into L2 ahead

// Phases of the batch-1 weight stream, in stream order within a layer; the LM head follows the
// last layer. QKV, GU and HEAD are row GEMVs (whole rows of W, a CTA owns a row range). OF and DF
// are folds: a CTA owns 8-column groups of Wo (its attention split's slice of the output) or of
// Wd (the gate/up pairs it computed), streamed as [group][d rows][8 columns], and adds
// W[:, its columns] * its inputs into the residual.
enum { PH_QKV = 0, PH_OF = 1, PH_GU = 2, PH_DF = 3, PH_HEAD = 4, KIE_NPH = 5 };

// Per-session sampling of the next token (top_k <= 1: greedy argmax).
struct SampleCfg {
    float inv_t;               // 1 / temperature
    int top_k;
    unsigned long long seed;
};
#define KIE_SAMPLE_VALS 6144   // values one CTA selects from in shared memory (batch-1 kernel)

// Commands of the resident kernel.
enum { OP_NONE = 0, OP_DECODE = 1, OP_PREFILL = 2, OP_TICK = 3, OP_EXIT = 4 };

// Device error codes (err word = code << 8 | where).
enum { DERR_BARRIER_TIMEOUT = 1, DERR_RING_TIMEOUT = 2, DERR_BAD_TOKEN = 3, DERR_MMA_TIMEOUT = 4, DERR_BOUNDS = 5 };

struct KieCmd {
    int32_t op, sid, pos0, n;
    int32_t in_tok;          // first input token of OP_DECODE
    int32_t n_sess;          // OP_TICK: sessions in the tick; OP_PREFILL on the tick kernel: rows
    uint32_t seq;            // doorbell sequence number
    int32_t flags;
    const int32_t *tokens;   // OP_PREFILL: input tokens [n] (device); OP_TICK: first inputs [n_sess]
    const int32_t *tok_dev;  // OP_DECODE via launch: device pointer to the first input token
    int32_t *out;            // output tokens (device memory or the mapped mailbox)
    float *logits;           // optional logits
    const int32_t *sids;     // OP_TICK: session ids [n_sess] (device)
    const int32_t *pos;      // OP_TICK: start positions [n_sess] (device)
};

// Host-mapped doorbell. The host writes `cmd`, then `cmd_seq`; the kernel writes the
// outputs, then `done_seq`.
struct KieMailbox {
    volatile uint32_t cmd_seq;
    uint32_t pad0[31];
    KieCmd cmd;
    uint32_t pad1[32 - (sizeof(KieCmd) / 4) % 32];
    volatile uint32_t done_seq;
    volatile int32_t status;
    uint32_t pad2[30];
    int32_t io[1];           // inputs then outputs (sized at allocation)
};

// Everything a kernel needs; passed by value.
struct KieParams {
    int L, d, Hq, Hkv, D, F, V, dtype, G;
    float eps;
    int max_ctx, max_sessions, nblk;
    int splits;                     // attention splits per kv head (batch-1)
    int cr[KIE_NPH];                // rows per ring chunk (GEMV phases) or 8-column groups per chunk (folds)
    int K[KIE_NPH];                 // row length (elements) per phase (8 for folds)
    // batch-1 packed weights: CTA c streams [seg_off[c], seg_off[c+1]) once per token
    const uint8_t *wpack;
    int wesz;                       // bytes per streamed weight: 2 (dtype), or 1 (E4M3 codes)
    int b1_tmem;                    // 1: ring chunks are moved on into TMEM and read from there
    int b1_kvr;                     // 1: the attention units' K/V rows stream through the weight ring
    const float *wsc;               // E4M3 row scales: per layer [QKV rows | d | gate/up rows | d], then [V]
    int sc_stride;                  // floats per layer in wsc
    const int *row0;                // [KIE_NPH][nblk+1] partition: rows (GEMV phases), 8-column groups (folds)
    const long long *seg_off;       // [nblk+1]
    // unpacked small weights
    const uint16_t *emb;            // [V][d]
    const uint16_t *gains;          // [2L+1][d]: attn_norm l, mlp_norm l, final
    const float2 *rope;             // [max_ctx][D/2] (cos, sin)
    // KV cache [sessions][L][Hkv][max_ctx][D]
    uint16_t *kcache, *vcache;
    long long sess_stride;
    // activations and scratch
    float *x, *q;                   // residual [d] (folds add into it), rotated queries [Hq*D]
    float *part;                    // [Hkv*splits*G][D+2]
    unsigned *cnt;                  // [Hkv]
    float *cand_val;
    int *cand_idx;                  // [nblk]
    const SampleCfg *samp;          // [max_sessions]
    float *cand_tv;                 // [nblk][KIE_TOPK_MAX] each CTA's top-k logits (sampling)
    int *cand_ti;                   // [nblk][KIE_TOPK_MAX] and their token ids
    int *tokbuf;                    // [max_ctx] device copy of command inputs
    unsigned long long *bar;        // grid barrier counter
    unsigned long long *rd;         // CTAs that have read the residual for the gate/up phase (split barrier)
    unsigned *err;                  // first device error
    KieMailbox *mbox;               // device alias of the mapped mailbox
    unsigned *last_seq;             // last doorbell sequence processed
    KieCmd *cmd;                    // command broadcast slot
    long long timeout_ns, idle_ns;
    unsigned long long *trace;      // phase stamps (null = off)
    int trace_tokens, trace_events;
    // multi-row (tick / chunked prefill) kernel: swizzled 128 x 64 weight tiles, CTA c streams
    // [mr_seg_off[c], mr_seg_off[c+1]); per GEMM phase it owns tiles [mr_a0[g][c], mr_a0[g][c+1])
    const uint8_t *mr_wpack;
    const long long *mr_seg_off;
    const int *mr_a0;               // [5][nblk+1]
    float *mr_x, *mr_yqkv, *mr_ygu, *mr_q, *mr_logits, *mr_part;
    // the B operand of the running GEMM: one swizzled 128 x 64 16-bit tile per k-step (rows
    // 0-63 hi, 64-127 lo of the activations), written by the phase that finalises them
    uint8_t *mr_bpack;
    // tensor maps (in device memory) of the K and V arenas viewed as [sessions * L * Hkv *
    // max_ctx][D], boxes of 128 rows x 64 dims with the 128-byte swizzle; null when D is not a
    // multiple of 64
    const void *mr_kmap, *mr_vmap;
    unsigned *mr_cnt;
    int *mr_sid, *mr_pos, *mr_tok;  // [64] rows of the current command
};

