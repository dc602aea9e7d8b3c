// Batch-1 decode megakernel for sm_100a.
//
// One CTA per SM stays resident across layers and tokens (the persistent single-kernel
// runtime of the HN digest of Kog's inference engine, section 技术原理, and the resident GPU
// program of "实时AI推理为何贵56倍？…", section 让工作常驻 GPU). A decode step streams every weight
// byte plus the KV cache once ("Kog 3000 tok/s 实时推理…", section 内存带宽优化的三层策略), so
// the kernel is organised around that stream:
//
//  * Warp 16 (the producer) walks this CTA's fixed weight schedule for the whole command
//    (all layers, all tokens) and copies it, chunk by chunk, into a 3 x 64 KB shared-memory
//    ring with 1-D bulk async copies (TMA). The schedule is contiguous in HBM because the
//    weights were repacked at engine creation in exactly this order, so each SM streams one
//    disjoint span (the aligned, topology-aware access of the same section). The producer
//    never waits on grid barriers.
//  * Warps 0-15 (consumers) run each layer as three phases, each ended by a grid barrier:
//      A  QKV : RMSNorm -> [Wq;Wk;Wv] rows -> RoPE -> q, and the K/V append to the cache
//      B  ATTN: split-K single-query attention; each split merges its slice of its kv head's
//               output (log-sum-exp), then folds it through its own columns of Wo into the
//               residual: x += Wo[:, slice] o[slice]
//      C  MLP : RMSNorm -> gate/up rows -> u = silu(gate) * up for this CTA's pairs, then the
//               same pairs' columns of Wd: x += Wd[:, pairs] u[pairs]
//    then, per token, HEAD: final RMSNorm -> LM-head rows -> block argmax -> grid argmax.
//    The two folds add into the residual with fp32 atomics, so no CTA has to wait for all of
//    o or u: that removes two of the five grid barriers a row-partitioned O and down
//    projection would need, and the gate/up and down weights stream back to back. In phase
//    C a CTA may add into x only after every CTA has read x for its RMSNorm: a split barrier
//    (arrive after the read, wait before the add) that is long complete when it is checked.
//
// GEMV mapping (QKV, gate/up, head): a ring chunk holds 2*CR whole rows of length K. The 16
// consumer warps form two groups of 8; group g takes rows [g*CR, (g+1)*CR) of every chunk.
// In a group, warp w owns the column slice [w*K/8, (w+1)*K/8); lane l owns 16-byte vectors
// l, l+32, ... of that slice, so a lane's slice of the input vector sits in registers for
// the whole phase and each staged weight byte is read from shared memory exactly once. Row
// sums are reduced across the warp with a shuffle butterfly over the CR rows; the 8
// column-slice partials of a row are added in a fixed order by the phase epilogue.
//
// Fold mapping (O and down): the CTA's columns arrive as [8-column group][d rows][8]
// (16 bytes per row and group); thread t owns rows t, t + 512, ... for the whole fold and
// accumulates them over its column groups, then adds them into x.
//
// RMSNorm: every CTA reads all of x for a normed phase, so each computes the sum of squares
// itself (one CTA-wide reduction) instead of publishing partial sums.
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kie_attn.cuh"
#include "kie_device.cuh"
#include "kie_sample.cuh"

namespace {

constexpr int RING_BYTES = KIE_NSLOT * KIE_SLOT_BYTES;

// ------------------------------------------------------------------ tensor memory (TMEM) staging
//
// With 16-bit weights and d_model 2048 or 4096, every 64 KB ring chunk gives each of the 512
// consumer threads exactly 8 pieces of 16 bytes (rows of its column slice, or rows of its fold
// columns), and within each piece index the 16-byte pieces of the warps' lanes lie at a uniform
// 16-byte stride, 512 bytes per warp. So the producer can move a landed chunk on from shared
// memory into one of 4 TMEM slots (128 columns each; all 512 columns of the SM) with 16
// tcgen05.cp copies of 128 lanes x 32 bytes that read the ring's own layout: copy j fills
// columns 8j..8j+7, i.e. pieces 2(j%4) and 2(j%4)+1 of warps 4(j/4) .. 4(j/4)+3, lane 32(w%4)+l
// holding thread (w, l)'s pieces. A consumer warp then takes its 8 pieces with one tcgen05.ld
// (32 lanes x 32 columns) of its lane quarter. The ring slot is free once the copies are done.
// The producer moves the chunks it fetches while the consumers are in the attention step and
// its grid barriers (produce_tmem), so there the weight stream runs 7 chunks (448 KB per SM)
// ahead of the consumers instead of 3.

constexpr uint32_t TMEM_COLS = 512;

KIE_DEV void tm_alloc(uint32_t *dst_smem) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
KIE_DEV void tm_dealloc(uint32_t taddr) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(TMEM_COLS) : "memory");
}
KIE_DEV void tm_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
KIE_DEV void tm_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// arrive on `bar` once every tcgen05 operation this thread issued so far has completed
KIE_DEV void tm_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// shared-memory descriptor, no swizzle: 8-row core matrices of 16-byte rows, `lbo` bytes between
// the two 16-byte halves of a 32-byte row, `sbo` bytes between consecutive 8-row groups
KIE_DEV uint64_t tm_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1u << 46);
}
KIE_DEV void tm_cp(uint32_t taddr, uint64_t desc) {
    asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}
// this warp's lane quarter, 32 consecutive columns -> 32 registers per thread
KIE_DEV void tm_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
KIE_DEV uint4 tm_piece(const uint32_t (&r)[32], int k) { return make_uint4(r[4 * k], r[4 * k + 1], r[4 * k + 2], r[4 * k + 3]); }

// byte offset in the ring chunk, and distance between the two 16-byte halves, of copy j (0..15)
// of a chunk of phase ph. GEMV chunks hold rows of d 16-bit weights: with d = 2048 piece k of
// warp w is row 8 (w / 8) + k of the chunk; with d = 4096 it is row 4 (w / 8) + k / 2, in column
// half k % 2 of the row (the halves 4096 bytes apart). Fold chunks: piece k is column group
// k / R, row tid + 512 (k % R), with R = d / 512 pieces per group.
KIE_DEV void tm_copy_src(int ph, int d, int j, uint32_t &off, uint32_t &lbo) {
    const uint32_t cg = (uint32_t)j >> 2, p = (uint32_t)j & 3u;
    if (ph == PH_OF || ph == PH_DF) {
        const uint32_t R = (uint32_t)d / 512u, k0 = 2u * p;
        off = (k0 / R) * (uint32_t)d * 16u + (k0 % R) * 8192u + cg * 2048u;
        lbo = 8192u;
    } else if (d == 2048) {
        off = ((cg >> 1) * 8u + 2u * p) * 4096u + (cg & 1u) * 2048u;
        lbo = 4096u;
    } else {
        off = ((cg >> 1) * 4u + p) * 8192u + (cg & 1u) * 2048u;
        lbo = 4096u;
    }
}

constexpr int WPART_FLOATS = 8 * KIE_ROWACC_MAX;  // column-slice partials: [slices][rows] flattened

// 8 streamed weights -> 8 floats: 16-byte vector of the storage dtype, or 8-byte vector of E4M3
// codes (element 0 in the lowest byte)
template <int DT, bool F8>
struct WVec;
template <int DT>
struct WVec<DT, false> {
    using T = uint4;
    static constexpr int BYTES = 16;
    static __device__ __forceinline__ void cvt(const T &w, float *f) { cvt8<DT>(w, f); }
};
template <int DT>
struct WVec<DT, true> {
    using T = uint2;
    static constexpr int BYTES = 8;
    static __device__ __forceinline__ void cvt(const T &w, float *f) {
        const uint32_t u[2] = {w.x, w.y};
#pragma unroll
        for (int j = 0; j < 2; j++) {
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(u[j] >> (16 * h)), __NV_E4M3);
                const float2 v = __half22float2(*reinterpret_cast<const __half2 *>(&r));
                f[4 * j + 2 * h] = v.x;
                f[4 * j + 2 * h + 1] = v.y;
            }
        }
    }
};

// offsets of a layer's phase blocks in the E4M3 row scales (P.wsc)
__device__ __forceinline__ int sc_off_o(const KieParams &P) { return (P.Hq + 2 * P.Hkv) * P.D; }
__device__ __forceinline__ int sc_off_gu(const KieParams &P) { return sc_off_o(P) + P.d; }
__device__ __forceinline__ int sc_off_down(const KieParams &P) { return sc_off_gu(P) + 2 * P.F; }

struct __align__(16) B1Shared {
    union {
        float wpart[WPART_FLOATS];  // column-slice partials of this phase's row sums
        struct {
            AttnSmem at;
            uint4 kvcur[2][KIE_DMAX / 8];       // K and V rows of the current position (last split)
        };
        struct {
            float vals[KIE_SAMPLE_VALS];  // the values a top-k selection reads
            SampleScratch ss;
        } samp;
    };
    float fold_in[KIE_FOLD_MAX];  // the current fold's inputs: this CTA's slice of o, or of u
    float red[64];
    int redi[32];
    float nrm[16];                // the RMSNorm's partial sums of squares (one per column slice)
    float2 rope_s[KIE_DMAX / 2];  // rotation of the current position, loaded at the start of QKV
    uint64_t full[KIE_NSLOT];
    uint64_t empty[KIE_NSLOT];
    uint64_t tfull[KIE_NTS];   // TMEM staging: slot t holds its chunk (tcgen05.commit)
    uint64_t tempty[KIE_NTS];  // every consumer warp has read slot t
    uint32_t tmem_base;
    uint32_t pub_sink;         // scratch word of pub_wait
    volatile uint32_t att_done;  // QKV -> attention barriers this CTA has passed in this launch
    KieCmd cmd;
    volatile int abort;
    int token;
    int gb_ok;
    int row0[KIE_NPH], row1[KIE_NPH];
    unsigned long long wait_ph[KIE_NPH];  // consumer ring waits of this token per phase (ns, traced runs)
    __align__(16) uint8_t warm_sink[512];  // destination of the K/V reads into L2 (16 bytes per lane; never read)
};

// word-wise copies of the command record (volatile: it may live in mapped host memory)
__device__ __forceinline__ void copy_words(KieCmd *dst, const KieCmd *src) {
    const volatile uint32_t *s = reinterpret_cast<const volatile uint32_t *>(src);
    uint32_t *d = reinterpret_cast<uint32_t *>(dst);
#pragma unroll
    for (int i = 0; i < (int)(sizeof(KieCmd) / 4); i++) d[i] = s[i];
}
__device__ __forceinline__ void copy_words_cg(KieCmd *dst, const KieCmd *src) {
    const uint32_t *s = reinterpret_cast<const uint32_t *>(src);
    uint32_t *d = reinterpret_cast<uint32_t *>(dst);
#pragma unroll
    for (int i = 0; i < (int)(sizeof(KieCmd) / 4); i++) d[i] = __ldcg(s + i);
}

// GEMV geometry fixed by the row length K: column slices per row (8: two warp groups take
// different rows of a chunk; 16: all warps share each row), 16-byte vectors per lane, and
// rows per group in one ring chunk. K <= 14336.
__host__ __device__ inline int col_slices(int K) { return K <= 8192 ? 8 : 16; }
__host__ __device__ inline int rows_per_group(int K) { return K <= 2048 ? 8 : K <= 4096 ? 4 : 2; }

__device__ __forceinline__ void trace_mark(const KieParams &P, int t, int ev, float after = 0.f) {
    if (P.trace && t < P.trace_tokens && threadIdx.x == 0 && in_bounds(ev < P.trace_events, P.err, 0x14))
        P.trace[((size_t)blockIdx.x * P.trace_tokens + t) * P.trace_events + ev] = globaltimer() + (after != after);
}

// --------------------------------------------------------------- grid barrier

// All consumer threads call this. Returns false if this CTA is aborting.
// fenced: the arrive is a release (the command broadcast, written with plain stores while no
// weight copies are in flight). Otherwise the values other CTAs read afterwards were published
// by completion (pub_*; every thread waited for them before the named barrier below), so the
// arrive is relaxed and does not wait for the weight stream's copies in flight.
__device__ bool grid_barrier(const KieParams &P, B1Shared &S, unsigned long long &epoch, long long timeout_ns,
                             unsigned where, bool fenced = false) {
    named_bar_sync(1, KIE_CONS_THREADS);
    if (threadIdx.x == 0) {
        int ok = !S.abort;
        if (ok) {
            epoch += 1;
            const unsigned long long target = epoch * (unsigned long long)P.nblk;
            if (fenced) red_release_gpu_add_u64(P.bar, 1ull);
            else red_relaxed_gpu_add_u64(P.bar, 1ull);
            uint64_t t0 = globaltimer();
            unsigned spins = 0;
            while (ld_acquire_gpu_u64(P.bar) < target) {
                if ((++spins & 255u) == 0) {
                    if (ld_volatile_u32(P.err) != 0u) {
                        ok = 0;
                        break;
                    }
                    if ((long long)(globaltimer() - t0) > timeout_ns) {
                        set_error(P.err, DERR_BARRIER_TIMEOUT, where);
                        ok = 0;
                        break;
                    }
                }
            }
            if (!ok) S.abort = 1;
        }
        S.gb_ok = ok;
    }
    named_bar_sync(1, KIE_CONS_THREADS);
    return S.gb_ok != 0;
}

// The split barrier of phase C. Thread 0 announces that this CTA has read the residual (the
// reads have returned: their values were used before the phase's last named barrier)...
__device__ __forceinline__ void residual_read_arrive(const KieParams &P, const B1Shared &S) {
    if (threadIdx.x == 0 && !S.abort) red_relaxed_gpu_add_u64(P.rd, 1ull);
}

// ... and before the first add into it waits until every CTA has done so (`epoch`: this
// CTA's arrivals so far, including the current one). All consumer threads call this.
__device__ void residual_read_wait(const KieParams &P, B1Shared &S, unsigned long long epoch) {
    if (threadIdx.x == 0 && !S.abort) {
        const unsigned long long target = epoch * (unsigned long long)P.nblk;
        const uint64_t t0 = globaltimer();
        unsigned spins = 0;
        while (ld_acquire_gpu_u64(P.rd) < target) {
            if ((++spins & 255u) == 0) {
                if (ld_volatile_u32(P.err) != 0u) {
                    S.abort = 1;
                    break;
                }
                if ((long long)(globaltimer() - t0) > P.timeout_ns) {
                    set_error(P.err, DERR_BARRIER_TIMEOUT, 7);
                    S.abort = 1;
                    break;
                }
            }
        }
    }
    named_bar_sync(1, KIE_CONS_THREADS);
}

// --------------------------------------------------------------- the weight schedule

// Walks this CTA's chunks in stream order: per token, every layer's QKV rows, O-fold column
// groups, gate/up rows and down-fold column groups, then (when the token needs logits) the
// LM-head rows. A token restarts at the segment base.
// K/V chunks (the attention unit's cache rows, when they stream through the ring) sit between
// a layer's QKV rows and its O-fold columns: positions [p0, p0 + n) of the unit's split other
// than the current one (final since earlier steps), KV_CHUNK_POS at a time, K rows at slot
// offset 0 and V rows at KIE_SLOT_BYTES / 2.
constexpr int PH_KV = KIE_NPH;
__host__ __device__ inline int kv_chunk_pos(int D) { return KIE_SLOT_BYTES / 4 / D; }
// query heads of a kv head the attention takes in one pass over the span (their queries and
// running sums are held in registers: the register budget of the 16 consumer warps allows two);
// more heads take more passes, each with the span streamed again
constexpr int ATT_GC = 2;
__host__ __device__ inline int kv_passes(const KieParams &P) { return (P.G + ATT_GC - 1) / ATT_GC; }

// The cache positions of this CTA's attention unit at context ctx that the ring carries:
// [p0, p0 + n), all of the split but the current position ctx - 1. false: no unit.
__device__ __forceinline__ bool kv_ring_span(const KieParams &P, int ctx, int &g, int &p0, int &n) {
    const int unit = blockIdx.x;
    if (unit >= P.Hkv * P.splits) return false;
    g = unit / P.splits;
    const int s = unit % P.splits;
    p0 = (int)((long long)s * ctx / P.splits);
    const int p1 = (int)((long long)(s + 1) * ctx / P.splits);
    n = max(0, min(p1, ctx - 1) - p0);
    return true;
}

struct ChunkIter {
    const uint8_t *seg, *g;
    int t, l, ph, r;
    int qn;  // chunks of this layer's O fold, gate/up and down fold returned so far
    int cq;  // the returned chunk's index among them (-1: a QKV, K/V or LM-head chunk)
    int kv_g, kv_p0, kv_n;  // K/V span of the current layer (PH_KV)
    int kv_pass;            // pass over the span (one per ATT_GC query heads)
};

__device__ __forceinline__ void chunk_begin(ChunkIter &it, const uint8_t *seg) {
    it.seg = seg;
    it.g = seg;
    it.t = 0;
    it.l = 0;
    it.ph = 0;
    it.r = 0;
    it.qn = 0;
    it.cq = -1;
}

__device__ __forceinline__ bool is_fold(int ph) { return ph == PH_OF || ph == PH_DF; }

// Next chunk (address, bytes); false when the command's schedule is exhausted. A GEMV chunk
// is cr rows of K elements; a fold chunk is cr column groups of d rows x 16 bytes; a K/V
// chunk is K rows at addr and as many V rows at addr2 (bytes covers both).
template <bool KVR>
__device__ bool chunk_next(const KieParams &P, const B1Shared &S, const KieCmd &cmd, ChunkIter &it,
                           const uint8_t *&addr, uint32_t &bytes, const uint8_t **addr2 = nullptr) {
    for (;;) {
        if (it.t >= cmd.n) return false;
        if (it.ph == PH_KV) {
            if (it.r < it.kv_n) {
                const int nr = min(kv_chunk_pos(P.D), it.kv_n - it.r);
                const size_t off = (size_t)cmd.sid * P.sess_stride +
                                   ((size_t)(it.l * P.Hkv + it.kv_g) * P.max_ctx + it.kv_p0 + it.r) * P.D;
                addr = reinterpret_cast<const uint8_t *>(P.kcache + off);
                if (addr2) *addr2 = reinterpret_cast<const uint8_t *>(P.vcache + off);
                bytes = (uint32_t)(2 * nr * P.D * 2);
                it.r += nr;
                it.cq = -1;
                return true;
            }
            it.r = 0;
            if (it.kv_n > 0 && ++it.kv_pass < kv_passes(P)) continue;  // the span again for the next query heads
            it.ph = PH_OF;
            continue;
        }
        const int n = S.row1[it.ph] - S.row0[it.ph];
        if (it.r < n) {
            const int nr = min(P.cr[it.ph], n - it.r);
            bytes = (uint32_t)(is_fold(it.ph) ? nr * P.d * 8 * P.wesz : nr * P.K[it.ph] * P.wesz);
            addr = it.g;
            it.g += bytes;
            it.r += nr;
            it.cq = (it.ph == PH_QKV || it.ph == PH_HEAD) ? -1 : it.qn++;
            return true;
        }
        // phase exhausted: advance
        it.r = 0;
        if (it.ph == PH_DF) it.qn = 0;
        if (it.ph == PH_HEAD) {
            it.t++;
            it.l = 0;
            it.ph = 0;
            it.g = it.seg;
        } else if (it.ph == PH_DF) {
            if (++it.l == P.L) {
                const bool head = (cmd.op != OP_PREFILL) || (it.t == cmd.n - 1);
                if (head) {
                    it.ph = PH_HEAD;
                } else {
                    it.t++;
                    it.l = 0;
                    it.ph = 0;
                    it.g = it.seg;
                }
            } else {
                it.ph = 0;
            }
        } else if (KVR && it.ph == PH_QKV) {
            it.ph = PH_KV;
            it.kv_pass = 0;
            if (!kv_ring_span(P, cmd.pos0 + it.t + 1, it.kv_g, it.kv_p0, it.kv_n)) it.kv_n = 0;
        } else {
            it.ph++;
        }
    }
}

// --------------------------------------------------------------- ring

// A consumer's wait for the data of ring slot `slot` (phase parity `par`). With the trace on,
// thread 0 adds the time it was blocked to the phase's total.
__device__ __forceinline__ bool ring_take(const KieParams &P, B1Shared &S, uint32_t slot, uint32_t par, int ph) {
    if (S.abort) return false;
    if (mbar_test_wait(&S.full[slot], par)) return true;
    const uint64_t w0 = globaltimer();
    const bool ok = mbar_wait(&S.full[slot], par, P.timeout_ns, &S.abort);
    if (P.trace && threadIdx.x == 0) S.wait_ph[ph] += globaltimer() - w0;
    return ok;
}

// The TMEM counterpart: wait until TMEM slot `ts` (phase parity `par`) holds its chunk.
__device__ __forceinline__ bool tmem_take(const KieParams &P, B1Shared &S, uint32_t ts, uint32_t par, int ph) {
    if (S.abort) return false;
    if (mbar_test_wait(&S.tfull[ts], par)) return true;
    const uint64_t w0 = globaltimer();
    const bool ok = mbar_wait(&S.tfull[ts], par, P.timeout_ns, &S.abort);
    if (P.trace && threadIdx.x == 0) S.wait_ph[ph] += globaltimer() - w0;
    return ok;
}

// A consumer warp's 8 pieces of the chunk in TMEM slot ts (see the staging layout above);
// the slot is released as soon as they are in registers.
__device__ __forceinline__ void tmem_read_chunk(B1Shared &S, uint32_t ts, uint32_t (&r)[32]) {
    const int w = threadIdx.x >> 5;
    tm_fence_after();
    tm_ld32(S.tmem_base + ((uint32_t)(32 * (w & 3)) << 16) + ts * 128u + 32u * (uint32_t)(w >> 2), r);
    tm_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&S.tempty[ts]);
}

// --------------------------------------------------------------- producer

// A K/V chunk of step t (t > 0 in the command), layer l, carries position pos - 1, which the
// previous step's QKV epilogues wrote in layer l: it may be copied once this CTA's consumers
// have passed that step's QKV -> attention barrier, the ((t - 1) L + l + 1)-th of the command
// (att0: barriers passed before the command). Earlier positions, and every position of step 0,
// were complete before. (With few chunks per step, as in small models, the stream can run
// that far ahead.)
__device__ __forceinline__ bool kv_chunk_ready(const KieParams &P, const B1Shared &S, const ChunkIter &it,
                                               uint32_t att0) {
    return it.t == 0 || (int)(S.att_done - (att0 + (uint32_t)((it.t - 1) * P.L + it.l + 1))) >= 0;
}

// Issues the bulk copies of one chunk into ring slot `slot`: a weight chunk in one piece, a K/V
// chunk as its K rows at the slot's start and its V rows at the slot's middle.
__device__ __forceinline__ void issue_chunk(B1Shared &S, uint8_t *ring, uint32_t slot, int ph, const uint8_t *a,
                                            const uint8_t *a2, uint32_t b) {
    uint8_t *dst = ring + (size_t)slot * KIE_SLOT_BYTES;
    mbar_arrive_expect_tx(&S.full[slot], b);
    if (ph == PH_KV) {
        bulk_g2s(dst, a, b / 2, &S.full[slot]);
        bulk_g2s(dst + KIE_SLOT_BYTES / 2, a2, b / 2, &S.full[slot]);
    } else {
        bulk_g2s(dst, a, b, &S.full[slot]);
    }
}

// Writes the producer's wait for this token into its trace slot.
__device__ __forceinline__ void trace_producer_wait(const KieParams &P, int tok, unsigned long long waited) {
    if (P.trace && tok < P.trace_tokens)
        P.trace[((size_t)blockIdx.x * P.trace_tokens + tok) * P.trace_events + P.trace_events - 1] = waited;
}

// Shared-memory ring only: chunk i goes to slot i % 3, and the consumers read it there.
template <bool KVR>
__device__ void produce_ring(const KieParams &P, B1Shared &S, uint32_t &ring_it, uint8_t *ring, const KieCmd &cmd) {
    const uint32_t att0 = S.att_done;
    const uint8_t *seg = P.wpack + P.seg_off[blockIdx.x];
    ChunkIter fetch;
    chunk_begin(fetch, seg);
    const uint8_t *a, *a2 = nullptr;
    uint32_t b;
    unsigned long long waited = 0;
    int tok = 0;
    while (chunk_next<KVR>(P, S, cmd, fetch, a, b, &a2)) {
        if (fetch.t != tok) {
            trace_producer_wait(P, tok, waited);
            waited = 0;
            tok = fetch.t;
        }
        const uint32_t slot = ring_it % KIE_NSLOT, par = (ring_it / KIE_NSLOT) & 1u;
        if (!mbar_test_wait(&S.empty[slot], par ^ 1u)) {
            const uint64_t w0 = globaltimer();
            const bool ok = !S.abort && mbar_wait(&S.empty[slot], par ^ 1u, P.timeout_ns, &S.abort);
            waited += globaltimer() - w0;
            if (!ok) {
                if (!S.abort) set_error(P.err, DERR_RING_TIMEOUT, 0x80);
                S.abort = 1;
                break;
            }
        }
        if (fetch.ph == PH_KV && !kv_chunk_ready(P, S, fetch, att0)) {
            const uint64_t w0 = globaltimer();
            while (!kv_chunk_ready(P, S, fetch, att0) && !S.abort) {
                if ((long long)(globaltimer() - w0) > P.timeout_ns) {
                    set_error(P.err, DERR_RING_TIMEOUT, 0x82);
                    S.abort = 1;
                }
                __nanosleep(64);
            }
            waited += globaltimer() - w0;
        }
        if (S.abort) break;
        issue_chunk(S, ring, slot, fetch.ph, a, a2, b);
        ring_it++;
    }
    trace_producer_wait(P, tok, waited);
    // Wait until every copy issued into the ring has landed before anyone may leave.
    const uint32_t first = ring_it > KIE_NSLOT ? ring_it - KIE_NSLOT : 0;
    for (uint32_t k = first; k < ring_it; k++)
        mbar_wait(&S.full[k % KIE_NSLOT], (k / KIE_NSLOT) & 1u, P.timeout_ns, nullptr);
}

// With TMEM staging, the first KIE_NTS chunks after each layer's QKV rows (its O-fold columns,
// then gate/up rows) move on from their ring slot into TMEM slot (m % KIE_NTS), m counting the
// moved chunks. Those are the chunks the producer fetches while the consumers are in the
// attention step and its grid barriers; moving them frees their ring slots for the next chunks,
// so the stream runs 7 chunks ahead there instead of 3. Every other chunk is read from the ring
// as without staging (the steady stream keeps its rate). A ring slot is free once its chunk
// has been read (16 consumer warps) or moved (the producer's 15 arrivals plus the copies'
// completion). Moves are issued in order; one waits for its chunk to land and for the
// consumers to be done with the TMEM slot's previous chunk, while the bulk copies run ahead.
__device__ __forceinline__ bool via_tmem(int cq) { return cq >= 0 && cq < KIE_NTS; }

template <bool KVR>
__device__ void produce_tmem(const KieParams &P, B1Shared &S, uint32_t &ring_it, uint32_t &tm_it, uint8_t *ring,
                             const KieCmd &cmd) {
    const uint32_t att0 = S.att_done;
    const uint8_t *seg = P.wpack + P.seg_off[blockIdx.x];
    ChunkIter fetch;
    chunk_begin(fetch, seg);
    const uint8_t *a = nullptr, *a2 = nullptr;
    uint32_t b = 0;
    bool more = chunk_next<KVR>(P, S, cmd, fetch, a, b, &a2);
    // moves waiting for their chunk to land or their TMEM slot: (chunk, phase), at most one per ring slot
    uint32_t mv_chunk[KIE_NSLOT];
    int mv_ph[KIE_NSLOT];
    int mv_n = 0, mv_head = 0;
    int tok = 0;
    unsigned long long waited = 0;
    uint64_t stall0 = 0;  // start of the current stall (0: making progress)
    const uint32_t ring_s = smem_u32(ring);
    const uint32_t tbase = S.tmem_base;
    while (more || mv_n > 0) {
        bool progress = false;
        if (more && (fetch.ph != PH_KV || kv_chunk_ready(P, S, fetch, att0))) {
            const uint32_t slot = ring_it % KIE_NSLOT, par = (ring_it / KIE_NSLOT) & 1u;
            if (mbar_test_wait(&S.empty[slot], par ^ 1u)) {
                if (fetch.t != tok) {
                    trace_producer_wait(P, tok, waited);
                    waited = 0;
                    tok = fetch.t;
                }
                issue_chunk(S, ring, slot, fetch.ph, a, a2, b);
                if (via_tmem(fetch.cq)) {
                    const int q = (mv_head + mv_n) % KIE_NSLOT;
                    mv_chunk[q] = ring_it;
                    mv_ph[q] = fetch.ph;
                    mv_n++;
                }
                ring_it++;
                more = chunk_next<KVR>(P, S, cmd, fetch, a, b, &a2);
                progress = true;
            }
        }
        if (mv_n > 0) {
            const uint32_t c = mv_chunk[mv_head];
            const uint32_t slot = c % KIE_NSLOT, par = (c / KIE_NSLOT) & 1u;
            const uint32_t ts = tm_it % KIE_NTS, tpar = (tm_it / KIE_NTS) & 1u;
            if (mbar_test_wait(&S.full[slot], par) && mbar_test_wait(&S.tempty[ts], tpar ^ 1u)) {
                tm_fence_after();
                const int ph = mv_ph[mv_head];
#pragma unroll 4
                for (int j = 0; j < 16; j++) {
                    uint32_t off, lbo;
                    tm_copy_src(ph, P.d, j, off, lbo);
                    tm_cp(tbase + ts * 128u + 8u * (uint32_t)j,
                          tm_desc(ring_s + slot * (uint32_t)KIE_SLOT_BYTES + off, lbo, 128u));
                }
                tm_commit(&S.tfull[ts]);
                tm_commit(&S.empty[slot]);                     // the last arrival: the copies are done
                mbar_arrive_n(&S.empty[slot], KIE_CONS_WARPS - 1);  // in place of the consumer warps
                tm_it++;
                mv_head = (mv_head + 1) % KIE_NSLOT;
                mv_n--;
                progress = true;
            }
        }
        if (progress) {
            if (stall0) waited += globaltimer() - stall0;
            stall0 = 0;
            continue;
        }
        const uint64_t now = globaltimer();
        if (!stall0) stall0 = now;
        if (S.abort) break;
        if ((long long)(now - stall0) > P.timeout_ns) {
            set_error(P.err, DERR_RING_TIMEOUT, 0x81);
            S.abort = 1;
            break;
        }
        // nothing to issue: sleep in hardware on the event most likely to come next (bounded, so
        // that the other stage is looked at again soon), leaving the issue slots to the consumers
        if (mv_n > 0) {
            const uint32_t c = mv_chunk[mv_head];
            if (!mbar_test_wait(&S.full[c % KIE_NSLOT], (c / KIE_NSLOT) & 1u))
                mbar_try_wait_ns(&S.full[c % KIE_NSLOT], (c / KIE_NSLOT) & 1u, 256);
            else
                mbar_try_wait_ns(&S.tempty[tm_it % KIE_NTS], ((tm_it / KIE_NTS) & 1u) ^ 1u, 256);
        } else if (more && fetch.ph == PH_KV) {
            __nanosleep(64);
        } else if (more) {
            mbar_try_wait_ns(&S.empty[ring_it % KIE_NSLOT], ((ring_it / KIE_NSLOT) & 1u) ^ 1u, 256);
        }
    }
    if (stall0) waited += globaltimer() - stall0;
    trace_producer_wait(P, tok, waited);
    // Before anyone may leave: every bulk copy issued has landed, and every move has completed
    // (a move's commit is the last arrival on its ring slot's empty barrier).
    for (uint32_t k = (ring_it > KIE_NSLOT ? ring_it - KIE_NSLOT : 0); k < ring_it; k++)
        mbar_wait(&S.full[k % KIE_NSLOT], (k / KIE_NSLOT) & 1u, P.timeout_ns, nullptr);
    for (uint32_t k = 0; k < KIE_NTS && k < tm_it; k++) {
        const uint32_t m = tm_it - 1 - k;
        mbar_wait(&S.tfull[m % KIE_NTS], (m / KIE_NTS) & 1u, P.timeout_ns, nullptr);
    }
}

// --------------------------------------------------------------- consumer: GEMV phases

// Runs one GEMV phase (QKV, gate/up or head) over this CTA's rows: the RMSNorm of its input
// (the embedding row at layer 0, else the residual x), then the rows; row partials land in
// S.wpart (see rowsum).
// With E4M3 weights, rsc receives the row scales the phase's epilogue applies: rows 2*tid and
// 2*tid + 1 of this CTA (the QKV and gate/up pairs), or rows tid and tid + 512 (head).
template <int DT, bool F8, bool TM, int NV, int CR, int CS>
__device__ void gemv_phase(const KieParams &P, B1Shared &S, uint32_t &ring_it, uint32_t &tm_it, int &lq,
                           const uint8_t *ring, int ph, int l, int tok, int pos, int t, float2 &rsc) {
    using WV = WVec<DT, F8>;
    constexpr int ESZ = F8 ? 1 : 2;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int K = P.K[ph];
    const int rows = S.row1[ph] - S.row0[ph];
    const bool from_emb = (ph == PH_QKV && l == 0);
    rsc = make_float2(1.f, 1.f);
    if (F8) {  // issued first: the loads complete under the row work
        const float *sc = P.wsc + (ph == PH_HEAD ? (size_t)P.L * P.sc_stride
                                                 : (size_t)l * P.sc_stride + (ph == PH_GU ? sc_off_gu(P) : 0)) + S.row0[ph];
        const int r0 = ph == PH_HEAD ? tid : 2 * tid, r1 = ph == PH_HEAD ? tid + KIE_CONS_THREADS : 2 * tid + 1;
        if (r0 < rows) rsc.x = __ldg(sc + r0);
        if (r1 < rows) rsc.y = __ldg(sc + r1);
    }

    // the QKV epilogue needs this position's rotation: fetch it now, under the row work
    if (ph == PH_QKV && tid < (P.D >> 1)) S.rope_s[tid] = P.rope[(size_t)pos * (P.D >> 1) + tid];
    const uint16_t *gain = P.gains + (size_t)(ph == PH_HEAD ? 2 * P.L : 2 * l + (ph == PH_GU ? 1 : 0)) * P.d;
    constexpr int GROUPS = KIE_CONS_WARPS / CS;  // warp groups, each taking CR rows of a chunk
    const int kslice = K / CS;  // columns per warp
    const int nvec = kslice >> 3;  // 16-byte vectors per warp slice
    float h[NV][8];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < NV; i++) {
        const int v = lane + 32 * i;
#pragma unroll
        for (int e = 0; e < 8; e++) h[i][e] = 0.f;
        if (v < nvec) {
            // 8 consecutive columns, 32-byte aligned. With TMEM staging and two vectors per lane,
            // vector i covers columns i K/2 + (w % CS) K/16 + 8 lane (the staging layout's column
            // halves); else the slice's columns in order.
            const int col0 = (TM && NV == 2) ? i * (K / 2) + (w % CS) * (K / 16) + 8 * lane : (w % CS) * kslice + 8 * v;
            if (from_emb) {
                cvt8<DT>(__ldg(reinterpret_cast<const uint4 *>(P.emb + (size_t)tok * P.d + col0)), h[i]);
            } else {
                const float4 a = __ldcg(reinterpret_cast<const float4 *>(P.x + col0));
                const float4 b = __ldcg(reinterpret_cast<const float4 *>(P.x + col0 + 4));
                h[i][0] = a.x; h[i][1] = a.y; h[i][2] = a.z; h[i][3] = a.w;
                h[i][4] = b.x; h[i][5] = b.y; h[i][6] = b.z; h[i][7] = b.w;
            }
            float g[8];
            cvt8<DT>(__ldg(reinterpret_cast<const uint4 *>(gain + col0)), g);
#pragma unroll
            for (int e = 0; e < 8; e++) {
                ss = fmaf(h[i][e], h[i][e], ss);
                h[i][e] *= g[e];
            }
        }
    }
    // 1/sqrt(mean(x^2) + eps) of the whole input: the CS warps of the first group cover every
    // column once; their sums are added in warp order after the rows, so every thread gets the
    // same value. It is one factor of every row sum, so the rows run on g * x and the factor
    // joins the row scales the epilogue applies (the reduction overlaps the first chunks).
    ss = warp_sum(ss);
    if (lane == 0 && w < CS) S.nrm[w] = ss;
    if (l < P.L) trace_mark(P, t, 1 + 16 * l + (ph == PH_QKV ? 11 : 12), h[0][0]);

    const int grp = w / CS, ws = w % CS;
    constexpr int STRIDE = WPART_FLOATS / CS;  // row capacity of one slice's partials
#ifdef KIE_PROFILE_GEMV
    // diagnostic build: SM cycles from a chunk's data being ready to this warp's release of
    // it, summed over the gate/up chunks, for the first warp of each row group
    long long busy = 0, c_ready = 0;
#endif
    // a chunk holds SUB blocks of GROUPS * CR rows (two with one-byte weights)
    constexpr int SUB = 2 / ESZ;
    constexpr int CH = SUB * GROUPS * CR;
    // with TMEM staging, the chunks among the layer's first KIE_NTS after its QKV rows were
    // moved into TMEM (lq: chunks of the layer seen so far; -1 for the QKV and head phases)
    int ntm = 0;
    if (TM && lq >= 0) {
        const int nch = (rows + CH - 1) / CH;
        ntm = min(max(KIE_NTS - lq, 0), nch);
        lq += nch;
    }
    // byte offset of vector i of this lane within a row: with TMEM staging and two vectors per
    // lane the staging layout's column halves, else the slice's columns in order
    auto colb = [&](int i) {
        return ((TM && NV == 2) ? i * (K / 2) + ws * (K / 16) + 8 * lane : ws * kslice + 8 * (lane + 32 * i)) * ESZ;
    };
    for (int c0 = 0, ci = 0; c0 < rows; c0 += CH, ci++) {
        const bool via = TM && ci < ntm;
        const uint32_t slot = ring_it % KIE_NSLOT, par = (ring_it / KIE_NSLOT) & 1u;
        const uint32_t ts = tm_it % KIE_NTS, tpar = (tm_it / KIE_NTS) & 1u;
        ring_it++;
        if (via) tm_it++;
        bool have = via ? tmem_take(P, S, ts, tpar, ph) : ring_take(P, S, slot, par, ph);
        have = __all_sync(0xffffffffu, have);  // one decision per warp (the reduction needs all lanes)
#ifdef KIE_PROFILE_GEMV
        c_ready = clock64();
#endif
        if (!have) {
            if (!S.abort) set_error(P.err, DERR_RING_TIMEOUT, (unsigned)ph);
            S.abort = 1;
            continue;  // keep the control flow; the command ends at the next barrier
        }
        if constexpr (TM) {
            if (via) {  // 16-bit weights: one block of GROUPS * CR rows; piece r NV + i is row r, vector i
                uint32_t tw[32];
                tmem_read_chunk(S, ts, tw);
                const int r0 = c0 + grp * CR;
                const int nr = max(0, min(CR, rows - r0));
                float acc[8];
#pragma unroll
                for (int r = 0; r < 8; r++) acc[r] = 0.f;
#pragma unroll
                for (int r = 0; r < CR; r++) {
                    if (r < nr) {
#pragma unroll
                        for (int i = 0; i < NV; i++) {
                            float f[8];
                            cvt8<DT>(tm_piece(tw, r * NV + i), f);
#pragma unroll
                            for (int e = 0; e < 8; e++) acc[r] = fmaf(f[e], h[i][e], acc[r]);
                        }
                    }
                }
                const float s = warp_reduce_rows<CR>(acc);
                constexpr int LPR = 32 / CR;
                if ((lane % LPR) == 0 && lane / LPR < nr) S.wpart[ws * STRIDE + r0 + lane / LPR] = s;
                continue;
            }
        }
#pragma unroll
        for (int sub = 0; sub < SUB; sub++) {
            const int r0 = c0 + (sub * GROUPS + grp) * CR;  // this group's first row in the block
            const int nr = max(0, min(CR, rows - r0));
            const uint8_t *base = ring + (size_t)slot * KIE_SLOT_BYTES + (size_t)(sub * GROUPS + grp) * CR * K * ESZ;
            float acc[8];
#pragma unroll
            for (int r = 0; r < 8; r++) acc[r] = 0.f;
#pragma unroll
            for (int r = 0; r < CR; r++) {
                if (r < nr) {
                    const uint8_t *rowp = base + (size_t)r * K * ESZ;
#pragma unroll
                    for (int i = 0; i < NV; i++) {
                        const int v = lane + 32 * i;
                        if (v < nvec) {
                            float f[8];
                            WV::cvt(*reinterpret_cast<const typename WV::T *>(rowp + colb(i)), f);
#pragma unroll
                            for (int e = 0; e < 8; e++) acc[r] = fmaf(f[e], h[i][e], acc[r]);
                        }
                    }
                }
            }
            if (sub == SUB - 1) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.empty[slot]);  // shared-memory reads of the chunk are done
#ifdef KIE_PROFILE_GEMV
                busy += clock64() - c_ready;
#endif
            }
            const float s = warp_reduce_rows<CR>(acc);
            constexpr int LPR = 32 / CR;
            if ((lane % LPR) == 0 && lane / LPR < nr) S.wpart[ws * STRIDE + r0 + lane / LPR] = s;
        }
    }
#ifdef KIE_PROFILE_GEMV
    if (P.trace && t < P.trace_tokens && l < P.L && ph == PH_GU && lane == 0 && ws == 0)
        P.trace[((size_t)blockIdx.x * P.trace_tokens + t) * P.trace_events + 1 + 16 * l + 13 + grp] = busy;
#endif
    named_bar_sync(1, KIE_CONS_THREADS);
    float tot = 0.f;
#pragma unroll
    for (int k = 0; k < CS; k++) tot += S.nrm[k];
    const float rstd = rsqrtf(tot / (float)P.d + P.eps);
    rsc.x *= rstd;
    rsc.y *= rstd;
}

// the row sum of row r of the current phase (column slices added in a fixed order)
__device__ __forceinline__ float rowsum(const B1Shared &S, int r, int cs) {
    float v = 0.f;
    const int stride = WPART_FLOATS / cs;
    for (int k = 0; k < cs; k++) v += S.wpart[k * stride + r];
    return v;
}

template <int DT, bool F8, bool TM>
__device__ __forceinline__ float2 gemv_dispatch(const KieParams &P, B1Shared &S, uint32_t &ring_it, uint32_t &tm_it,
                                                int &lq, const uint8_t *ring, int ph, int l, int tok, int pos, int t) {
    const int K = P.K[ph];
    float2 rsc;
    if (K <= 2048) gemv_phase<DT, F8, TM, 1, 8, 8>(P, S, ring_it, tm_it, lq, ring, ph, l, tok, pos, t, rsc);
    else gemv_phase<DT, F8, TM, 2, 4, 8>(P, S, ring_it, tm_it, lq, ring, ph, l, tok, pos, t, rsc);  // K <= 4096
    return rsc;
}

// --------------------------------------------------------------- consumer: folds

// One fold (O or down): this CTA's 8-column groups of W arrive as [group][d rows][8], and
// S.fold_in holds 8 inputs per group. Thread t accumulates rows t + 512 j over all groups.
template <int DT, bool F8, bool TM, int RPT>
__device__ void fold_rows(const KieParams &P, B1Shared &S, uint32_t &ring_it, uint32_t &tm_it, int &lq,
                          const uint8_t *ring, int ph, float (&acc)[RPT]) {
    using WV = WVec<DT, F8>;
    const int tid = threadIdx.x, lane = tid & 31;
    const int d = P.d, ng = S.row1[ph] - S.row0[ph], cpc = P.cr[ph];
#pragma unroll
    for (int j = 0; j < RPT; j++) acc[j] = 0.f;
    named_bar_sync(1, KIE_CONS_THREADS);  // S.fold_in was written by other warps of this CTA
    int ntm = 0;  // leading chunks staged in TMEM (see gemv_phase)
    if (TM && lq >= 0) {
        const int nch = (ng + cpc - 1) / cpc;
        ntm = min(max(KIE_NTS - lq, 0), nch);
        lq += nch;
    }
    for (int g0 = 0, ci = 0; g0 < ng; g0 += cpc, ci++) {
        const int n = min(cpc, ng - g0);
        const bool via = TM && ci < ntm;
        const uint32_t slot = ring_it % KIE_NSLOT, par = (ring_it / KIE_NSLOT) & 1u;
        const uint32_t ts = tm_it % KIE_NTS, tpar = (tm_it / KIE_NTS) & 1u;
        ring_it++;
        if (via) tm_it++;
        bool have = via ? tmem_take(P, S, ts, tpar, ph) : ring_take(P, S, slot, par, ph);
        have = __all_sync(0xffffffffu, have);
        if (!have) {
            if (!S.abort) set_error(P.err, DERR_RING_TIMEOUT, (unsigned)ph);
            S.abort = 1;
            continue;
        }
        if (TM && via) {
            // the chunk's cpc = 8 / RPT column groups: piece k = gi RPT + j is row tid + 512 j of group gi
            uint32_t tw[32];
            tmem_read_chunk(S, ts, tw);
#pragma unroll
            for (int gi = 0; gi < 8 / RPT; gi++) {
                if (gi < n) {
                    const float4 a = *reinterpret_cast<const float4 *>(&S.fold_in[(g0 + gi) * 8]);
                    const float4 b = *reinterpret_cast<const float4 *>(&S.fold_in[(g0 + gi) * 8 + 4]);
                    const float in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int j = 0; j < RPT; j++) {
                        float f[8];
                        cvt8<DT>(tm_piece(tw, gi * RPT + j), f);
#pragma unroll
                        for (int e = 0; e < 8; e++) acc[j] = fmaf(f[e], in[e], acc[j]);
                    }
                }
            }
        } else {
            const uint8_t *base = ring + (size_t)slot * KIE_SLOT_BYTES;
            for (int gi = 0; gi < n; gi++) {
                const float4 a = *reinterpret_cast<const float4 *>(&S.fold_in[(g0 + gi) * 8]);
                const float4 b = *reinterpret_cast<const float4 *>(&S.fold_in[(g0 + gi) * 8 + 4]);
                const float in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int j = 0; j < RPT; j++) {
                    const int r = tid + KIE_CONS_THREADS * j;
                    if (r < d) {
                        float f[8];
                        WV::cvt(*reinterpret_cast<const typename WV::T *>(base + ((size_t)gi * d + r) * WV::BYTES), f);
#pragma unroll
                        for (int e = 0; e < 8; e++) acc[j] = fmaf(f[e], in[e], acc[j]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.empty[slot]);
        }
    }
}

// x[r] += acc (times the row's scale with E4M3 weights) for this thread's rows (fp32 atomics:
// the folds of all CTAs meet in x)
template <int RPT>
__device__ __forceinline__ void fold_commit(const KieParams &P, B1Shared &S, const float (&acc)[RPT], int ph,
                                            const float (&scl)[RPT]) {
    if (S.abort || S.row1[ph] == S.row0[ph]) return;
    uint32_t tok = 0;
#pragma unroll
    for (int j = 0; j < RPT; j++) {
        const int r = threadIdx.x + KIE_CONS_THREADS * j;
        if (r < P.d) pub_add_f32(P.x + r, acc[j] * scl[j], tok);
    }
    pub_wait(tok, &S.pub_sink);  // the next grid barrier's arrive follows these adds' completion
}

// the fold's row scales (E4M3 weights), loaded before the fold so they arrive under its work
template <bool F8, int RPT>
__device__ __forceinline__ void fold_scales(const KieParams &P, int l, int off, float (&scl)[RPT]) {
#pragma unroll
    for (int j = 0; j < RPT; j++) {
        const int r = threadIdx.x + KIE_CONS_THREADS * j;
        scl[j] = (F8 && r < P.d) ? __ldg(P.wsc + (size_t)l * P.sc_stride + off + r) : 1.f;
    }
}

// --------------------------------------------------------------- consumer: epilogues

__device__ __forceinline__ void attention_prefetch(const KieParams &P, B1Shared &S, int l, int sid, int pos);

// q/k rows come in rotation pairs (dim i, dim i + D/2); v rows use the same pairing. Thread p
// takes pair p (npair <= 512); the CTA's pairs come two at a time as dims (i, i + 1), i even, of
// one head, so the even thread of each two writes both dims as one word (q: two fp32 values,
// k and v: two 16-bit values), published by completion for the attention step.
template <int DT, bool KVR>
__device__ void epilogue_qkv(const KieParams &P, B1Shared &S, int l, int sid, int pos, int tok, float2 rsc) {
    const int D = P.D, half = D >> 1, qd = P.Hq * D, kvd = P.Hkv * D;
    const int rbeg = S.row0[PH_QKV], npair = (S.row1[PH_QKV] - rbeg) >> 1;
    const size_t sess = (size_t)sid * P.sess_stride;
    const int p = threadIdx.x;
    const int r = rbeg + 2 * p;
    const int i = (r % D) >> 1;
    const bool act = p < npair;
    float ra = 0.f, rb = 0.f;
    if (act) {
        const int cs = col_slices(P.K[PH_QKV]);
        const float a = rowsum(S, 2 * p, cs) * rsc.x, b = rowsum(S, 2 * p + 1, cs) * rsc.y;
        if (r < qd + kvd) {  // rotate q and k
            const float2 c = S.rope_s[i];
            ra = a * c.x - b * c.y;
            rb = b * c.x + a * c.y;
        } else {
            ra = a;
            rb = b;
        }
    }
    const float ra1 = __shfl_down_sync(0xffffffffu, ra, 1), rb1 = __shfl_down_sync(0xffffffffu, rb, 1);
    uint32_t tk = 0;
    if (act && (p & 1) == 0) {
        auto pack = [](float x0, float x1) { return (uint32_t)store1<DT>(x0) | ((uint32_t)store1<DT>(x1) << 16); };
        if (r < qd) {
            float *qp = P.q + (r / D) * D;
            if (in_bounds((r / D) * D + i + half + 1 < qd, P.err, 0x10)) {
                pub_f32x2(qp + i, ra, ra1, tk);
                pub_f32x2(qp + i + half, rb, rb1, tk);
            }
        } else {
            const bool isk = r < qd + kvd;
            const int g = (r - qd - (isk ? 0 : kvd)) / D;
            uint16_t *cp = (isk ? P.kcache : P.vcache) + sess + ((size_t)(l * P.Hkv + g) * P.max_ctx + pos) * D;
            if (in_bounds(pos < P.max_ctx && g < P.Hkv && sid < P.max_sessions && i + half + 1 < D, P.err, 0x11)) {
                pub_u32(cp + i, pack(ra, ra1), tk);
                pub_u32(cp + i + half, pack(rb, rb1), tk);
            }
        }
    }
    if (l == 0) {  // the residual starts as the embedding row (each CTA writes a 1/nblk share)
        const int r0 = (int)((long long)blockIdx.x * P.d / P.nblk), r1 = (int)((long long)(blockIdx.x + 1) * P.d / P.nblk);
        for (int rr = r0 + threadIdx.x; rr < r1; rr += KIE_CONS_THREADS) pub_f32(P.x + rr, cvt1<DT>(P.emb[(size_t)tok * P.d + rr]), tk);
        if (!KVR) attention_prefetch(P, S, l, sid, pos);
    }
    pub_wait(tk, &S.pub_sink);
}

// The cache rows this CTA's attention unit will read in layer l are read into L2 ahead of
// time (older positions are final; L2 stays coherent for the one written in this token).
__device__ __forceinline__ void attention_prefetch(const KieParams &P, B1Shared &S, int l, int sid, int pos) {
    const int D = P.D;
    const size_t sess = (size_t)sid * P.sess_stride;
    const int ctx = pos + 1;
    for (int unit = blockIdx.x; unit < P.Hkv * P.splits; unit += P.nblk) {
        const int g = unit / P.splits, s = unit % P.splits;
        const long long p0 = (long long)s * ctx / P.splits, p1 = (long long)(s + 1) * ctx / P.splits;
        const size_t off = sess + ((size_t)(l * P.Hkv + g) * P.max_ctx + p0) * D;
        // whole lines (a partial one is left to the loads), at most 256 KB per unit: at long
        // contexts a layer's cache outgrows L2, and reading it all ahead would evict itself and
        // compete with the weight stream of the phase that issues the reads
        const int lines = (int)min((p1 - p0) * D * 2 / 128, (long long)KIE_KV_WARM_LINES);
        for (int j = threadIdx.x; j < 2 * lines; j += KIE_CONS_THREADS) {
            const uint16_t *base = (j < lines ? P.kcache : P.vcache) + off;
            l2_warm_line(S.warm_sink + (threadIdx.x & 31) * 16, reinterpret_cast<const uint8_t *>(base) + (size_t)(j % lines) * 128);
        }
    }
}

// u = silu(gate) * up for this CTA's pairs, into the down fold's inputs
template <bool KVR>
__device__ void epilogue_gu(const KieParams &P, B1Shared &S, int l, int sid, int pos, float2 rsc) {
    if (!KVR && l + 1 < P.L) attention_prefetch(P, S, l + 1, sid, pos);
    const int npair = (S.row1[PH_GU] - S.row0[PH_GU]) >> 1;
    const int cs = col_slices(P.K[PH_GU]);
    for (int p = threadIdx.x; p < npair; p += KIE_CONS_THREADS) {
        const float g = rowsum(S, 2 * p, cs) * rsc.x, up = rowsum(S, 2 * p + 1, cs) * rsc.y;  // (p == tid)
        S.fold_in[p] = g / (1.f + expf(-g)) * up;
    }
}

__device__ __forceinline__ void argmax_combine(float &v, int &i, float v2, int i2) {
    if (v2 > v || (v2 == v && i2 < i)) {
        v = v2;
        i = i2;
    }
}

__device__ void warp_argmax(float &v, int &i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
        argmax_combine(v, i, v2, i2);
    }
}

// logits of this CTA's rows -> optional output, local argmax -> candidate slot
__device__ void epilogue_head(const KieParams &P, B1Shared &S, float *logits, float2 rsc) {
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int rbeg = S.row0[PH_HEAD], n = S.row1[PH_HEAD] - rbeg;
    float bv = -CUDART_INF_F;
    int bi = 0x7fffffff;
    for (int r = tid; r < n; r += KIE_CONS_THREADS) {  // rows tid and tid + 512 (n <= 1024)
        const float v = rowsum(S, r, col_slices(P.K[PH_HEAD])) * (r == tid ? rsc.x : rsc.y);
        if (logits && in_bounds(rbeg + r < P.V, P.err, 0x12)) logits[rbeg + r] = v;
        argmax_combine(bv, bi, v, rbeg + r);
    }
    warp_argmax(bv, bi);
    if (lane == 0) {
        S.red[w] = bv;
        S.redi[w] = bi;
    }
    named_bar_sync(1, KIE_CONS_THREADS);
    if (w == 0) {
        float v = lane < KIE_CONS_WARPS ? S.red[lane] : -CUDART_INF_F;
        int i = lane < KIE_CONS_WARPS ? S.redi[lane] : 0x7fffffff;
        warp_argmax(v, i);
        if (lane == 0) {  // published by completion for the head's grid barrier
            uint32_t tk = 0;
            pub_f32(P.cand_val + blockIdx.x, v, tk);
            pub_u32(P.cand_idx + blockIdx.x, (uint32_t)i, tk);
            pub_wait(tk, &S.pub_sink);
        }
    }
}

// after the head barrier: every warp of every CTA reduces all candidates to the same
// token, so no further barrier is needed
__device__ int final_argmax(const KieParams &P) {
    const int lane = threadIdx.x & 31;
    float v = -CUDART_INF_F;
    int i = 0x7fffffff;
    for (int c = lane; c < P.nblk; c += 32) argmax_combine(v, i, __ldcg(P.cand_val + c), __ldcg(P.cand_idx + c));
    warp_argmax(v, i);
    return i;
}

// Sampling head, first stage: this CTA's logits (rows rbeg .. rbeg + n) -> optional output,
// then its top-k (value, token) into the candidate slots cand_tv/cand_ti[cta][0..k); slots past
// the CTA's row count hold NaN, which ranks below every number.
// (Arguments by value: a reference to the kernel's parameter block would make the kernel keep
// a copy of it in local memory.)
__device__ __noinline__ void sample_local(B1Shared &S, float *logits, int k, int cs, float *cand_tv, int *cand_ti,
                                          int V, float2 rsc) {
    const int tid = threadIdx.x;
    const int rbeg = S.row0[PH_HEAD], n = S.row1[PH_HEAD] - rbeg;
    float v0 = 0.f, v1 = 0.f;  // rows tid and tid + 512 (n <= 1024)
    if (tid < n) v0 = rowsum(S, tid, cs) * rsc.x;
    if (tid + KIE_CONS_THREADS < n) v1 = rowsum(S, tid + KIE_CONS_THREADS, cs) * rsc.y;
    if (logits) {
        if (tid < n) logits[rbeg + tid] = v0;
        if (tid + KIE_CONS_THREADS < n) logits[rbeg + tid + KIE_CONS_THREADS] = v1;
    }
    named_bar_sync(1, KIE_CONS_THREADS);  // the row partials are read: their space takes the values
    if (tid < n) S.samp.vals[tid] = v0;
    if (tid + KIE_CONS_THREADS < n) S.samp.vals[tid + KIE_CONS_THREADS] = v1;
    const int kl = min(k, n);
    if (kl > 0) {
        const float *vals = S.samp.vals;
        block_topk<KIE_CONS_THREADS>(S.samp.ss, n, kl, [&](int p) { return vals[p]; }, [&](int p) { return rbeg + p; });
    } else {
        named_bar_sync(1, KIE_CONS_THREADS);
    }
    if (tid < KIE_TOPK_MAX) {  // published by completion for the head's grid barrier
        const bool have = tid < kl;
        uint32_t tk = 0;
        pub_f32(cand_tv + blockIdx.x * KIE_TOPK_MAX + tid, have ? S.samp.ss.top_v[tid] : CUDART_NAN_F, tk);
        pub_u32(cand_ti + blockIdx.x * KIE_TOPK_MAX + tid, (uint32_t)(have ? S.samp.ss.top_i[tid] : V + tid), tk);
        pub_wait(tk, &S.pub_sink);
    }
}

// Sampling head, second stage (after the head barrier, in every CTA): the top-k of all CTAs'
// candidates (CTA c's at positions c*k .. c*k + k - 1: equal values keep the token order), the
// draw of position pos, the token. Returns the same token in every thread.
__device__ __noinline__ int sample_global(B1Shared &S, int nblk, const float *cand_tv, const int *cand_ti, float inv_t,
                                         int k, unsigned long long seed, int pos) {
    const int tid = threadIdx.x, n = nblk * k;
    for (int p = tid; p < n; p += KIE_CONS_THREADS)
        S.samp.vals[p] = __ldcg(cand_tv + (p / k) * KIE_TOPK_MAX + p % k);
    named_bar_sync(1, KIE_CONS_THREADS);
    const float *vals = S.samp.vals;
    const int *ti = cand_ti;
    block_topk<KIE_CONS_THREADS>(S.samp.ss, n, k, [&](int p) { return vals[p]; },
                                 [&](int p) { return __ldcg(ti + (p / k) * KIE_TOPK_MAX + p % k); });
    if (tid < 32) {
        const int tok = sample_pick(S.samp.ss, k, inv_t, sample_uniform(seed, pos));
        if (tid == 0) S.token = tok;
    }
    named_bar_sync(1, KIE_CONS_THREADS);
    const int tok = S.token;
    named_bar_sync(1, KIE_CONS_THREADS);  // S.token is read before anyone reuses the space
    return tok;
}

// --------------------------------------------------------------- consumer: attention

// The QKV -> attention barrier, then this CTA's attention unit (at most one unit per CTA:
// splits = nblk / Hkv); the query heads of a kv head are taken GC at a time. Each split merges
// its slice of the kv head's output into S.fold_in (the O fold's inputs).
// This CTA's attention unit (kv head g, split s) for query heads [hoff, hoff + GC) of the kv
// head: its cache rows arrive through the weight ring (positions [p0, p0 + n) of the split, in
// chunks of kv_chunk_pos(D) positions, one pass of the span per GC query heads), and in the
// last split the current position's row, written this step by the QKV epilogues and published
// before the barrier, is read from the cache at the start and taken last by position group 0.
// Then the split merge (attn_tail). Position groups of D/8 lanes, scores in log2 units, as in
// attn_unit.
template <int DT, int GC>
__device__ void attn_unit_ring(const KieParams &P, B1Shared &S, const AttnArgs &A, uint32_t &ring_it,
                               const uint8_t *ring, int ctx, int hoff) {
    constexpr int NW = KIE_CONS_WARPS;
    constexpr int B = 1;  // positions per group per batch (registers)
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int D = P.D, lpp = D >> 3, ppw = 32 / lpp, sub = lane / lpp, sl = lane % lpp;
    const int ngroups = NW * ppw, gi = w * ppw + sub;
    const int Gt = P.G, nh = min(GC, Gt - hoff);
    const float qscale = rsqrtf((float)D) * 1.4426950408889634f;
    int g, p0, n;
    kv_ring_span(P, ctx, g, p0, n);  // the caller checked that this CTA has a unit
    const bool last = (int)blockIdx.x % P.splits == P.splits - 1;
    float q[GC][8];
#pragma unroll
    for (int jj = 0; jj < GC; jj++) {
        const float *qp = P.q + (size_t)(g * Gt + hoff + min(jj, nh - 1)) * D + sl * 8;
        const float4 a = __ldcg(reinterpret_cast<const float4 *>(qp));
        const float4 b = __ldcg(reinterpret_cast<const float4 *>(qp + 4));
        q[jj][0] = a.x * qscale; q[jj][1] = a.y * qscale; q[jj][2] = a.z * qscale; q[jj][3] = a.w * qscale;
        q[jj][4] = b.x * qscale; q[jj][5] = b.y * qscale; q[jj][6] = b.z * qscale; q[jj][7] = b.w * qscale;
    }
    // the current position's K and V rows (last split), staged for position group 0
    if (last && tid < 2 * (D / 8)) {
        const int kvsel = tid / (D / 8), c = tid % (D / 8);
        const size_t o = (size_t)g * A.head_stride + (size_t)(ctx - 1) * D + c * 8;
        S.kvcur[kvsel][c] = __ldcg(reinterpret_cast<const uint4 *>((kvsel ? A.v : A.k) + o));
    }
    named_bar_sync(1, KIE_CONS_THREADS);
    float m[GC], lsum[GC], acc[GC][8];
#pragma unroll
    for (int jj = 0; jj < GC; jj++) {
        m[jj] = -CUDART_INF_F;
        lsum[jj] = 0.f;
#pragma unroll
        for (int e = 0; e < 8; e++) acc[jj][e] = 0.f;
    }
    const int PB = kv_chunk_pos(D);
    for (int c0 = 0; c0 < n; c0 += PB) {
        const int np = min(PB, n - c0);
        const uint32_t slot = ring_it % KIE_NSLOT, par = (ring_it / KIE_NSLOT) & 1u;
        ring_it++;
        bool have = ring_take(P, S, slot, par, PH_OF);  // traced with the O fold's waits
        have = __all_sync(0xffffffffu, have);
        if (!have) {
            if (!S.abort) set_error(P.err, DERR_RING_TIMEOUT, (unsigned)PH_KV);
            S.abort = 1;
            continue;
        }
        const uint8_t *kb = ring + (size_t)slot * KIE_SLOT_BYTES, *vb = kb + KIE_SLOT_BYTES / 2;
        for (int base = 0; base < np; base += ngroups * B) {  // uniform across the CTA
            uint4 kv[B], vv[B];
#pragma unroll
            for (int b = 0; b < B; b++) {
                const int j = base + gi + b * ngroups;
                const bool ok = j < np;
                const size_t o = ((size_t)j * D + sl * 8) * 2;
                kv[b] = ok ? *reinterpret_cast<const uint4 *>(kb + o) : make_uint4(0, 0, 0, 0);
                vv[b] = ok ? *reinterpret_cast<const uint4 *>(vb + o) : make_uint4(0, 0, 0, 0);
            }
            attn_update<DT, GC, B>(kv, vv, base, np, gi, ngroups, lpp, q, m, lsum, acc);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[slot]);
    }
    if (last) {
        uint4 kv[1], vv[1];
        kv[0] = gi == 0 ? S.kvcur[0][sl] : make_uint4(0, 0, 0, 0);
        vv[0] = gi == 0 ? S.kvcur[1][sl] : make_uint4(0, 0, 0, 0);
        attn_update<DT, GC, 1>(kv, vv, 0, 1, gi, ngroups, lpp, q, m, lsum, acc);
    }
    attn_tail<DT, GC, NW, false>(A, S.at, (int)blockIdx.x, Gt, hoff, m, lsum, acc);
}

template <int DT, int GC, bool KVR>
__device__ void attention_step(const KieParams &P, B1Shared &S, int l, int sid, int pos, unsigned long long &epoch,
                               int t, int e, uint32_t &att_use, uint32_t &ring_it, const uint8_t *ring) {
    AttnArgs A;
    A.q = P.q;
    A.k = P.kcache + (size_t)sid * P.sess_stride + (size_t)l * P.Hkv * P.max_ctx * P.D;
    A.v = P.vcache + (size_t)sid * P.sess_stride + (size_t)l * P.Hkv * P.max_ctx * P.D;
    A.head_stride = (long long)P.max_ctx * P.D;
    A.part = P.part;
    A.cnt = P.cnt;
    A.o = nullptr;
    A.bpack = nullptr;
    A.brow = 0;
    A.gout = -1;
    // every split merges a slice once all splits of its kv head have published; each split
    // adds one per pass over the query heads, and the counters only count up within a launch
    A.cnt_target = (att_use + 1u) * (uint32_t)P.splits * (uint32_t)((P.G + GC - 1) / GC);
    A.oslice = S.fold_in;
    A.timeout_ns = P.timeout_ns;
    A.err = P.err;
    att_use++;
    A.D = P.D;
    A.Hkv = P.Hkv;
    A.nsplit = P.splits;
    A.ctx = pos + 1;
    const int unit = blockIdx.x;
    const bool have = unit < P.Hkv * P.splits;
    grid_barrier(P, S, epoch, P.timeout_ns, 1);
    if (threadIdx.x == 0) S.att_done = S.att_done + 1u;  // this step's K/V rows are complete (see kv_chunk_ready)
    trace_mark(P, t, e + 2);
    if (P.wesz == 1)  // the O fold's row scales (E4M3 weights) wait in L1 through attention
        for (int r = threadIdx.x; r < P.d; r += KIE_CONS_THREADS)
            prefetch_l1(P.wsc + (size_t)l * P.sc_stride + sc_off_o(P) + r);
    if (threadIdx.x == 0) S.at.t_unit = 0;
    if (have && !S.abort) {
        for (int hoff = 0; hoff < P.G; hoff += GC) {
            if constexpr (KVR) attn_unit_ring<DT, GC>(P, S, A, ring_it, ring, pos + 1, hoff);
            else attn_unit<DT, GC, KIE_CONS_WARPS>(A, S.at, unit, P.G, hoff);  // K/V from L2 (read ahead)
        }
    }
}

// the two folds of a layer and the down fold's split barrier, by rows per thread
template <int DT, bool F8, bool TM, int RPT>
__device__ __forceinline__ void o_fold(const KieParams &P, B1Shared &S, uint32_t &ring_it, uint32_t &tm_it, int &lq,
                                       const uint8_t *ring, int l) {
    float acc[RPT], scl[RPT];
    fold_scales<F8, RPT>(P, l, sc_off_o(P), scl);
    fold_rows<DT, F8, TM, RPT>(P, S, ring_it, tm_it, lq, ring, PH_OF, acc);
    fold_commit<RPT>(P, S, acc, PH_OF, scl);
}

template <int DT, bool F8, bool TM, int RPT>
__device__ __forceinline__ void down_fold(const KieParams &P, B1Shared &S, uint32_t &ring_it, uint32_t &tm_it, int &lq,
                                          const uint8_t *ring, int l, unsigned long long rd_epoch, int t, int e) {
    float acc[RPT], scl[RPT];
    fold_scales<F8, RPT>(P, l, sc_off_down(P), scl);
    fold_rows<DT, F8, TM, RPT>(P, S, ring_it, tm_it, lq, ring, PH_DF, acc);
    residual_read_wait(P, S, rd_epoch);  // every CTA has read x for its gate/up norm
    trace_mark(P, t, e + 10);
    fold_commit<RPT>(P, S, acc, PH_DF, scl);
}

// rows per thread of a fold (d <= 4096): 1, 2, 4 or 8
template <int DT, bool F8, bool TM>
__device__ __forceinline__ void o_fold_any(const KieParams &P, B1Shared &S, uint32_t &ring_it, uint32_t &tm_it,
                                           int &lq, const uint8_t *ring, int l) {
    if constexpr (TM) {  // d is 2048 or 4096
        if (P.d <= 2048) o_fold<DT, F8, TM, 4>(P, S, ring_it, tm_it, lq, ring, l);
        else o_fold<DT, F8, TM, 8>(P, S, ring_it, tm_it, lq, ring, l);
        return;
    }
    if (P.d <= 512) o_fold<DT, F8, TM, 1>(P, S, ring_it, tm_it, lq, ring, l);
    else if (P.d <= 1024) o_fold<DT, F8, TM, 2>(P, S, ring_it, tm_it, lq, ring, l);
    else if (P.d <= 2048) o_fold<DT, F8, TM, 4>(P, S, ring_it, tm_it, lq, ring, l);
    else o_fold<DT, F8, TM, 8>(P, S, ring_it, tm_it, lq, ring, l);
}

template <int DT, bool F8, bool TM>
__device__ __forceinline__ void down_fold_any(const KieParams &P, B1Shared &S, uint32_t &ring_it, uint32_t &tm_it,
                                              int &lq, const uint8_t *ring, int l, unsigned long long rd_epoch, int t,
                                              int e) {
    if constexpr (TM) {  // d is 2048 or 4096
        if (P.d <= 2048) down_fold<DT, F8, TM, 4>(P, S, ring_it, tm_it, lq, ring, l, rd_epoch, t, e);
        else down_fold<DT, F8, TM, 8>(P, S, ring_it, tm_it, lq, ring, l, rd_epoch, t, e);
        return;
    }
    if (P.d <= 512) down_fold<DT, F8, TM, 1>(P, S, ring_it, tm_it, lq, ring, l, rd_epoch, t, e);
    else if (P.d <= 1024) down_fold<DT, F8, TM, 2>(P, S, ring_it, tm_it, lq, ring, l, rd_epoch, t, e);
    else if (P.d <= 2048) down_fold<DT, F8, TM, 4>(P, S, ring_it, tm_it, lq, ring, l, rd_epoch, t, e);
    else down_fold<DT, F8, TM, 8>(P, S, ring_it, tm_it, lq, ring, l, rd_epoch, t, e);
}

// --------------------------------------------------------------- consumer: one command

template <int DT, bool F8, bool TM, bool KVR>
__device__ void consume(const KieParams &P, B1Shared &S, uint32_t &ring_it, uint32_t &tm_it, const uint8_t *ring,
                        const KieCmd &cmd, unsigned long long &epoch, unsigned long long &rd_epoch, uint32_t &att_use) {
    int tok = cmd.in_tok;
    if (cmd.op == OP_DECODE && cmd.tok_dev) tok = __ldcg(cmd.tok_dev);
    const int L = P.L;
    SampleCfg sc;
    sc.inv_t = __ldcg(&P.samp[cmd.sid].inv_t);
    sc.top_k = __ldcg(&P.samp[cmd.sid].top_k);
    sc.seed = __ldcg(&P.samp[cmd.sid].seed);
    for (int t = 0; t < cmd.n; t++) {
        const int pos = cmd.pos0 + t;
        if (cmd.op == OP_PREFILL) tok = __ldcg(P.tokbuf + t);
        if (tok < 0 || tok >= P.V) {
            // e.g. a caller's device token, or an argmax over non-finite logits: fail the
            // command, and read no row outside the embedding table on the way out
            if (threadIdx.x == 0) set_error(P.err, DERR_BAD_TOKEN, 0);
            S.abort = 1;
            tok = 0;
        }
        if (threadIdx.x < KIE_NPH) S.wait_ph[threadIdx.x] = 0;
        trace_mark(P, t, 0);
        const bool head = (cmd.op != OP_PREFILL) || (t == cmd.n - 1);
        for (int l = 0; l < L; l++) {
            const int e = 1 + 16 * l;
            // A: QKV
            int lq = -1;  // the QKV rows are never staged in TMEM
            const float2 sq = gemv_dispatch<DT, F8, TM>(P, S, ring_it, tm_it, lq, ring, PH_QKV, l, tok, pos, t);
            lq = 0;  // the chunks of the O fold, gate/up rows and down fold, counted from here
            trace_mark(P, t, e);
            epilogue_qkv<DT, KVR>(P, S, l, cmd.sid, pos, tok, sq);
            trace_mark(P, t, e + 1);
            // B: attention, then the O fold
            attention_step<DT, ATT_GC, KVR>(P, S, l, cmd.sid, pos, epoch, t, e, att_use, ring_it, ring);
            if (P.trace && t < P.trace_tokens && threadIdx.x == 0)  // end of this CTA's positions (0: no unit)
                P.trace[((size_t)blockIdx.x * P.trace_tokens + t) * P.trace_events + e + 15] = S.at.t_unit;
            trace_mark(P, t, e + 3);
            o_fold_any<DT, F8, TM>(P, S, ring_it, tm_it, lq, ring, l);
            trace_mark(P, t, e + 4);
            grid_barrier(P, S, epoch, P.timeout_ns, 2);
            trace_mark(P, t, e + 5);
            // C: gate/up, then the down fold
            const float2 sg = gemv_dispatch<DT, F8, TM>(P, S, ring_it, tm_it, lq, ring, PH_GU, l, tok, pos, t);
            residual_read_arrive(P, S);  // this CTA's reads of x are done
            rd_epoch++;
            trace_mark(P, t, e + 6);
            epilogue_gu<KVR>(P, S, l, cmd.sid, pos, sg);
            trace_mark(P, t, e + 7);
            down_fold_any<DT, F8, TM>(P, S, ring_it, tm_it, lq, ring, l, rd_epoch, t, e);
            trace_mark(P, t, e + 8);
            grid_barrier(P, S, epoch, P.timeout_ns, 3);
            trace_mark(P, t, e + 9);
        }
        const int eh = 1 + 16 * L;
        if (head) {
            int lq = -1;
            const float2 sh = gemv_dispatch<DT, F8, TM>(P, S, ring_it, tm_it, lq, ring, PH_HEAD, L, tok, pos, t);
            float *lg = nullptr;
            if (cmd.logits) lg = cmd.logits + (cmd.op == OP_PREFILL ? 0 : (size_t)t * P.V);
            if (sc.top_k > 1) sample_local(S, lg, sc.top_k, col_slices(P.K[PH_HEAD]), P.cand_tv, P.cand_ti, P.V, sh);
            else epilogue_head(P, S, lg, sh);
            trace_mark(P, t, eh);
            grid_barrier(P, S, epoch, P.timeout_ns, 6);
            trace_mark(P, t, eh + 1);
            tok = sc.top_k > 1 ? sample_global(S, P.nblk, P.cand_tv, P.cand_ti, sc.inv_t, sc.top_k, sc.seed, pos)
                               : final_argmax(P);
            if (blockIdx.x == 0 && threadIdx.x == 0) {
                if (cmd.out) cmd.out[cmd.op == OP_PREFILL ? 0 : t] = tok;
                // no index wins an argmax over non-finite logits: the command fails (a later
                // step of it also stops at the token check above)
                if (tok < 0 || tok >= P.V) set_error(P.err, DERR_BAD_TOKEN, 1);
            }
            trace_mark(P, t, eh + 2);
        }
        if (P.trace && t < P.trace_tokens && threadIdx.x < KIE_NPH)
            P.trace[((size_t)blockIdx.x * P.trace_tokens + t) * P.trace_events + P.trace_events - 1 - KIE_NPH +
                    threadIdx.x] = S.wait_ph[threadIdx.x];
    }
    if (!KVR) cp_async_wait_all();  // the L2 reads into warm_sink have landed
}

// --------------------------------------------------------------- the kernel

template <int DT, bool F8, bool TM, bool KVR>
__global__ void __launch_bounds__(KIE_THREADS, 1) kie_b1_kernel(KieParams P, KieCmd one, int resident) {
    extern __shared__ __align__(1024) uint8_t smem[];
    B1Shared &S = *reinterpret_cast<B1Shared *>(smem + RING_BYTES);
    const int tid = threadIdx.x;
    if (tid == 0) {
        for (int i = 0; i < KIE_NSLOT; i++) {
            mbar_init(&S.full[i], 1);
            // a chunk's 16 consumer warps, or (moved into TMEM) the producer's 15 arrivals and
            // the commit of the copies
            mbar_init(&S.empty[i], KIE_CONS_WARPS);
        }
        for (int i = 0; i < KIE_NTS; i++) {
            mbar_init(&S.tfull[i], 1);
            mbar_init(&S.tempty[i], KIE_CONS_WARPS);
        }
        fence_mbar_init();
        S.abort = 0;
        S.att_done = 0;
    }
    if (tid < KIE_NPH) {
        S.row0[tid] = P.row0[tid * (P.nblk + 1) + blockIdx.x];
        S.row1[tid] = P.row0[tid * (P.nblk + 1) + blockIdx.x + 1];
    }
    if (TM && tid < 32) tm_alloc(&S.tmem_base);  // all 512 columns (one CTA per SM); freed at exit
    tm_fence_before();
    __syncthreads();
    tm_fence_after();
    uint32_t ring_it = 0;  // chunks consumed (consumers) / issued (producer); both advance identically
    uint32_t tm_it = 0;    // chunks staged in TMEM, counted the same way on both sides
    unsigned long long epoch = 0;
    unsigned long long rd_epoch = 0;  // split-barrier arrivals of this CTA so far in this launch
    uint32_t att_use = 0;  // attention phases so far in this launch (the merge counters' targets)
    for (;;) {
        if (tid < KIE_CONS_THREADS) {
            if (!resident) {
                if (tid == 0) S.cmd = one;
            } else {
                // the doorbell: CTA 0 waits for the host's next command and broadcasts it
                if (blockIdx.x == 0) {
                    if (tid == 0) {
                        const unsigned last = *P.last_seq;
                        const uint64_t t0 = globaltimer();
                        KieCmd c{};
                        c.op = OP_EXIT;
                        for (;;) {
                            const uint32_t s = ld_acquire_sys_u32(&P.mbox->cmd_seq);
                            if (s != last) {
                                copy_words(&c, &P.mbox->cmd);
                                c.seq = s;
                                *P.last_seq = s;
                                break;
                            }
                            if ((long long)(globaltimer() - t0) > P.idle_ns) break;
                            __nanosleep(256);
                        }
                        *P.cmd = c;
                        S.cmd = c;
                    }
                    named_bar_sync(1, KIE_CONS_THREADS);
                    // a prompt arrives in the mailbox; stage it in device memory for all CTAs
                    if (S.cmd.op == OP_PREFILL)
                        for (int j = tid; j < S.cmd.n; j += KIE_CONS_THREADS)
                            if (in_bounds(j < P.max_ctx, P.err, 0x13)) P.tokbuf[j] = ((const volatile int32_t *)S.cmd.tokens)[j];
                }
                grid_barrier(P, S, epoch, P.idle_ns + P.timeout_ns, 0, true);
                if (tid == 0) {
                    copy_words_cg(&S.cmd, P.cmd);
                    if (S.abort) S.cmd.op = OP_EXIT;
                }
            }
        }
        __syncthreads();
        const KieCmd cmd = S.cmd;
        if (cmd.op != OP_DECODE && cmd.op != OP_PREFILL) break;
        if (tid >= KIE_CONS_THREADS) {
            if (tid == KIE_CONS_THREADS) {
                if constexpr (TM) produce_tmem<KVR>(P, S, ring_it, tm_it, smem, cmd);
                else produce_ring<KVR>(P, S, ring_it, smem, cmd);
            }
        } else {
            consume<DT, F8, TM, KVR>(P, S, ring_it, tm_it, smem, cmd, epoch, rd_epoch, att_use);
        }
        __syncthreads();
        if (resident && blockIdx.x == 0 && tid == 0) {
            __threadfence_system();
            P.mbox->status = (S.abort || ld_volatile_u32(P.err) != 0u) ? -1 : 0;
            st_release_sys_u32(&P.mbox->done_seq, cmd.seq);
        }
        if (!resident || S.abort) break;
    }
    if constexpr (TM) {  // every move has completed and every consumer read has returned
        tm_fence_before();
        __syncthreads();
        tm_fence_after();
        if (tid < 32) tm_dealloc(S.tmem_base);
    }
}

}  // namespace

// --------------------------------------------------------------- host-side launch helpers

extern "C++" {

size_t kie_b1_smem_bytes() { return RING_BYTES + sizeof(B1Shared); }

// rows per ring chunk for row length K, and the most rows one CTA may own in such a phase
int kie_b1_chunk_rows(int K) { return (KIE_CONS_WARPS / col_slices(K)) * rows_per_group(K); }
int kie_b1_max_rows(int K) { return WPART_FLOATS / col_slices(K); }

// TMEM staging needs the layouts its copies assume: 16-bit weights, d_model 2048 or 4096
bool kie_b1_tmem_ok(int d, bool f8) { return !f8 && (d == 2048 || d == 4096); }

// the kernel instantiation for a storage dtype, weight format, staging and K/V path
template <int DT>
static const void *b1_fn_dt(bool f8, bool tm, bool kvr) {
    if (f8) return kvr ? (const void *)kie_b1_kernel<DT, true, false, true> : (const void *)kie_b1_kernel<DT, true, false, false>;
    if (tm) return kvr ? (const void *)kie_b1_kernel<DT, false, true, true> : (const void *)kie_b1_kernel<DT, false, true, false>;
    return kvr ? (const void *)kie_b1_kernel<DT, false, false, true> : (const void *)kie_b1_kernel<DT, false, false, false>;
}
static const void *b1_fn(int dtype, bool f8, bool tm, bool kvr) {
    return dtype == KIE_BF16 ? b1_fn_dt<KIE_BF16>(f8, tm, kvr) : b1_fn_dt<KIE_FP16>(f8, tm, kvr);
}

cudaError_t kie_b1_prepare(int dtype, bool f8, bool tm, bool kvr) {
    return cudaFuncSetAttribute(b1_fn(dtype, f8, tm, kvr), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kie_b1_smem_bytes());
}

cudaError_t kie_b1_occupancy(int dtype, bool f8, bool tm, bool kvr, int *blocks_per_sm) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, b1_fn(dtype, f8, tm, kvr), KIE_THREADS,
                                                         kie_b1_smem_bytes());
}

cudaError_t kie_b1_launch(const KieParams &P, const KieCmd &one, int resident, cudaStream_t stream) {
    // the attention merge counters count up from zero within a launch
    const cudaError_t e = cudaMemsetAsync(P.cnt, 0, (size_t)P.Hkv * sizeof(unsigned), stream);
    if (e != cudaSuccess) return e;
    KieParams p = P;
    KieCmd c = one;
    int r = resident;
    void *args[] = {&p, &c, &r};
    return cudaLaunchCooperativeKernel(b1_fn(P.dtype, P.wesz == 1, P.b1_tmem != 0, P.b1_kvr != 0), dim3(P.nblk), dim3(KIE_THREADS), args,
                                       kie_b1_smem_bytes(), stream);
}

}  // extern "C++"
