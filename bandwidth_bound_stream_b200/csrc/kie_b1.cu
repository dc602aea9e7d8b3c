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
        AttnSmem at;
        struct {
            float vals[KIE_SAMPLE_VALS];  // the values a top-k selection reads
            SampleScratch ss;
        } samp;
    };
    float fold_in[KIE_FOLD_MAX];  // the current fold's inputs: this CTA's slice of o, or of u
    float red[64];
    int redi[32];
    float2 rope_s[KIE_DMAX / 2];  // rotation of the current position, loaded at the start of QKV
    uint64_t full[KIE_NSLOT];
    uint64_t empty[KIE_NSLOT];
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
    if (P.trace && t < P.trace_tokens && threadIdx.x == 0)
        P.trace[((size_t)blockIdx.x * P.trace_tokens + t) * P.trace_events + ev] = globaltimer() + (after != after);
}

// --------------------------------------------------------------- grid barrier

// All consumer threads call this. Returns false if this CTA is aborting.
__device__ bool grid_barrier(const KieParams &P, B1Shared &S, unsigned long long &epoch, long long timeout_ns,
                             unsigned where) {
    named_bar_sync(1, KIE_CONS_THREADS);
    if (threadIdx.x == 0) {
        int ok = !S.abort;
        if (ok) {
            epoch += 1;
            const unsigned long long target = epoch * (unsigned long long)P.nblk;
            // release: this CTA's writes (ordered before by the named barrier) become visible
            red_release_gpu_add_u64(P.bar, 1ull);
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

// The split barrier of phase C. Thread 0 announces that this CTA has read the residual (its
// earlier reads are ordered before the release)...
__device__ __forceinline__ void residual_read_arrive(const KieParams &P, const B1Shared &S) {
    if (threadIdx.x == 0 && !S.abort) red_release_gpu_add_u64(P.rd, 1ull);
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
struct ChunkIter {
    const uint8_t *seg, *g;
    int t, l, ph, r;
};

__device__ __forceinline__ void chunk_begin(ChunkIter &it, const uint8_t *seg) {
    it.seg = seg;
    it.g = seg;
    it.t = 0;
    it.l = 0;
    it.ph = 0;
    it.r = 0;
}

__device__ __forceinline__ bool is_fold(int ph) { return ph == PH_OF || ph == PH_DF; }

// Next chunk (address, bytes); false when the command's schedule is exhausted. A GEMV chunk
// is cr rows of K elements; a fold chunk is cr column groups of d rows x 16 bytes.
__device__ bool chunk_next(const KieParams &P, const B1Shared &S, const KieCmd &cmd, ChunkIter &it,
                           const uint8_t *&addr, uint32_t &bytes) {
    for (;;) {
        if (it.t >= cmd.n) return false;
        const int n = S.row1[it.ph] - S.row0[it.ph];
        if (it.r < n) {
            const int nr = min(P.cr[it.ph], n - it.r);
            bytes = (uint32_t)(is_fold(it.ph) ? nr * P.d * 8 * P.wesz : nr * P.K[it.ph] * P.wesz);
            addr = it.g;
            it.g += bytes;
            it.r += nr;
            return true;
        }
        // phase exhausted: advance
        it.r = 0;
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

// --------------------------------------------------------------- producer

__device__ void produce(const KieParams &P, B1Shared &S, uint32_t &ring_it, uint8_t *ring, const KieCmd &cmd) {
    const uint8_t *seg = P.wpack + P.seg_off[blockIdx.x];
    ChunkIter fetch;
    chunk_begin(fetch, seg);
    const uint8_t *a;
    uint32_t b;
    unsigned long long waited = 0;
    int tok = 0;
    while (chunk_next(P, S, cmd, fetch, a, b)) {
        if (fetch.t != tok) {
            if (P.trace && tok < P.trace_tokens)
                P.trace[((size_t)blockIdx.x * P.trace_tokens + tok) * P.trace_events + P.trace_events - 1] = waited;
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
        if (S.abort) break;
        mbar_arrive_expect_tx(&S.full[slot], b);
        bulk_g2s(ring + (size_t)slot * KIE_SLOT_BYTES, a, b, &S.full[slot]);
        ring_it++;
    }
    if (P.trace && tok < P.trace_tokens)
        P.trace[((size_t)blockIdx.x * P.trace_tokens + tok) * P.trace_events + P.trace_events - 1] = waited;
    // Wait until every copy issued into the ring has landed before anyone may leave.
    const uint32_t first = ring_it > KIE_NSLOT ? ring_it - KIE_NSLOT : 0;
    for (uint32_t k = first; k < ring_it; k++)
        mbar_wait(&S.full[k % KIE_NSLOT], (k / KIE_NSLOT) & 1u, P.timeout_ns, nullptr);
}

// --------------------------------------------------------------- consumer: GEMV phases

// Runs one GEMV phase (QKV, gate/up or head) over this CTA's rows: the RMSNorm of its input
// (the embedding row at layer 0, else the residual x), then the rows; row partials land in
// S.wpart (see rowsum).
// With E4M3 weights, rsc receives the row scales the phase's epilogue applies: rows 2*tid and
// 2*tid + 1 of this CTA (the QKV and gate/up pairs), or rows tid and tid + 512 (head).
template <int DT, bool F8, int NV, int CR, int CS>
__device__ void gemv_phase(const KieParams &P, B1Shared &S, uint32_t &ring_it, const uint8_t *ring, int ph, int l,
                           int tok, int pos, int t, float2 &rsc) {
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
            const int col0 = (w % CS) * kslice + 8 * v;  // 8 consecutive columns, 32-byte aligned
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
    // column once; their sums are added in warp order, so every thread gets the same value
    ss = warp_sum(ss);
    if (lane == 0 && w < CS) S.red[w] = ss;
    named_bar_sync(1, KIE_CONS_THREADS);
    float tot = 0.f;
#pragma unroll
    for (int k = 0; k < CS; k++) tot += S.red[k];
    const float rstd = rsqrtf(tot / (float)P.d + P.eps);
#pragma unroll
    for (int i = 0; i < NV; i++)
#pragma unroll
        for (int e = 0; e < 8; e++) h[i][e] *= rstd;
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
    for (int c0 = 0; c0 < rows; c0 += SUB * GROUPS * CR) {
        const uint32_t slot = ring_it % KIE_NSLOT, par = (ring_it / KIE_NSLOT) & 1u;
        ring_it++;
        bool have = ring_take(P, S, slot, par, ph);
        have = __all_sync(0xffffffffu, have);  // one decision per warp (the reduction needs all lanes)
#ifdef KIE_PROFILE_GEMV
        c_ready = clock64();
#endif
        if (!have) {
            if (!S.abort) set_error(P.err, DERR_RING_TIMEOUT, (unsigned)ph);
            S.abort = 1;
            continue;  // keep the control flow; the command ends at the next barrier
        }
#pragma unroll
        for (int sub = 0; sub < SUB; sub++) {
            const int r0 = c0 + (sub * GROUPS + grp) * CR;  // this group's first row in the block
            const int nr = max(0, min(CR, rows - r0));
            const uint8_t *base = ring + (size_t)slot * KIE_SLOT_BYTES +
                                  ((size_t)(sub * GROUPS + grp) * CR * K + (size_t)ws * kslice) * ESZ;
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
                            WV::cvt(*reinterpret_cast<const typename WV::T *>(rowp + v * WV::BYTES), f);
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
}

// the row sum of row r of the current phase (column slices added in a fixed order)
__device__ __forceinline__ float rowsum(const B1Shared &S, int r, int cs) {
    float v = 0.f;
    const int stride = WPART_FLOATS / cs;
    for (int k = 0; k < cs; k++) v += S.wpart[k * stride + r];
    return v;
}

template <int DT, bool F8>
__device__ __forceinline__ float2 gemv_dispatch(const KieParams &P, B1Shared &S, uint32_t &ring_it, const uint8_t *ring,
                                                int ph, int l, int tok, int pos, int t) {
    const int K = P.K[ph];
    float2 rsc;
    if (K <= 2048) gemv_phase<DT, F8, 1, 8, 8>(P, S, ring_it, ring, ph, l, tok, pos, t, rsc);
    else gemv_phase<DT, F8, 2, 4, 8>(P, S, ring_it, ring, ph, l, tok, pos, t, rsc);  // K <= 4096
    return rsc;
}

// --------------------------------------------------------------- consumer: folds

// One fold (O or down): this CTA's 8-column groups of W arrive as [group][d rows][8], and
// S.fold_in holds 8 inputs per group. Thread t accumulates rows t + 512 j over all groups.
template <int DT, bool F8, int RPT>
__device__ void fold_rows(const KieParams &P, B1Shared &S, uint32_t &ring_it, const uint8_t *ring, int ph,
                          float (&acc)[RPT]) {
    using WV = WVec<DT, F8>;
    const int tid = threadIdx.x, lane = tid & 31;
    const int d = P.d, ng = S.row1[ph] - S.row0[ph], cpc = P.cr[ph];
#pragma unroll
    for (int j = 0; j < RPT; j++) acc[j] = 0.f;
    named_bar_sync(1, KIE_CONS_THREADS);  // S.fold_in was written by other warps of this CTA
    for (int g0 = 0; g0 < ng; g0 += cpc) {
        const int n = min(cpc, ng - g0);
        const uint32_t slot = ring_it % KIE_NSLOT, par = (ring_it / KIE_NSLOT) & 1u;
        ring_it++;
        bool have = ring_take(P, S, slot, par, ph);
        have = __all_sync(0xffffffffu, have);
        if (!have) {
            if (!S.abort) set_error(P.err, DERR_RING_TIMEOUT, (unsigned)ph);
            S.abort = 1;
            continue;
        }
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

// x[r] += acc (times the row's scale with E4M3 weights) for this thread's rows (fp32 atomics:
// the folds of all CTAs meet in x)
template <int RPT>
__device__ __forceinline__ void fold_commit(const KieParams &P, const B1Shared &S, const float (&acc)[RPT], int ph,
                                            const float (&scl)[RPT]) {
    if (S.abort || S.row1[ph] == S.row0[ph]) return;
#pragma unroll
    for (int j = 0; j < RPT; j++) {
        const int r = threadIdx.x + KIE_CONS_THREADS * j;
        if (r < P.d) atomicAdd(P.x + r, acc[j] * scl[j]);
    }
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

// q/k rows come in rotation pairs (dim i, dim i + D/2); v rows use the same pairing.
template <int DT>
__device__ void epilogue_qkv(const KieParams &P, B1Shared &S, int l, int sid, int pos, int tok, float2 rsc) {
    const int D = P.D, half = D >> 1, qd = P.Hq * D, kvd = P.Hkv * D;
    const int rbeg = S.row0[PH_QKV], npair = (S.row1[PH_QKV] - rbeg) >> 1;
    const size_t sess = (size_t)sid * P.sess_stride;
    for (int p = threadIdx.x; p < npair; p += KIE_CONS_THREADS) {
        const int r = rbeg + 2 * p;
        const int cs = col_slices(P.K[PH_QKV]);
        const float a = rowsum(S, 2 * p, cs) * rsc.x, b = rowsum(S, 2 * p + 1, cs) * rsc.y;  // (p == tid)
        const int i = (r % D) >> 1;
        if (r < qd + kvd) {
            const float2 cs = S.rope_s[i];
            const float ra = a * cs.x - b * cs.y, rb = b * cs.x + a * cs.y;
            if (r < qd) {
                const int hh = r / D;
                P.q[hh * D + i] = ra;
                P.q[hh * D + i + half] = rb;
            } else {
                const int g = (r - qd) / D;
                uint16_t *kp = P.kcache + sess + ((size_t)(l * P.Hkv + g) * P.max_ctx + pos) * D;
                kp[i] = store1<DT>(ra);
                kp[i + half] = store1<DT>(rb);
            }
        } else {
            const int g = (r - qd - kvd) / D;
            uint16_t *vp = P.vcache + sess + ((size_t)(l * P.Hkv + g) * P.max_ctx + pos) * D;
            vp[i] = store1<DT>(a);
            vp[i + half] = store1<DT>(b);
        }
    }
    if (l == 0) {  // the residual starts as the embedding row (each CTA writes a 1/nblk share)
        const int r0 = (int)((long long)blockIdx.x * P.d / P.nblk), r1 = (int)((long long)(blockIdx.x + 1) * P.d / P.nblk);
        for (int r = r0 + threadIdx.x; r < r1; r += KIE_CONS_THREADS) P.x[r] = cvt1<DT>(P.emb[(size_t)tok * P.d + r]);
        attention_prefetch(P, S, l, sid, pos);
    }
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
__device__ void epilogue_gu(const KieParams &P, B1Shared &S, int l, int sid, int pos, float2 rsc) {
    if (l + 1 < P.L) attention_prefetch(P, S, l + 1, sid, pos);
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
        if (logits) logits[rbeg + r] = v;
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
        if (lane == 0) {
            P.cand_val[blockIdx.x] = v;
            P.cand_idx[blockIdx.x] = i;
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
    if (tid < KIE_TOPK_MAX) {
        const bool have = tid < kl;
        cand_tv[blockIdx.x * KIE_TOPK_MAX + tid] = have ? S.samp.ss.top_v[tid] : CUDART_NAN_F;
        cand_ti[blockIdx.x * KIE_TOPK_MAX + tid] = have ? S.samp.ss.top_i[tid] : V + tid;
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
template <int DT, int GC>
__device__ void attention_step(const KieParams &P, B1Shared &S, int l, int sid, int pos, unsigned long long &epoch,
                               int t, int e, uint32_t &att_use) {
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
    trace_mark(P, t, e + 2);
    if (P.wesz == 1)  // the O fold's row scales (E4M3 weights) wait in L1 through attention
        for (int r = threadIdx.x; r < P.d; r += KIE_CONS_THREADS)
            prefetch_l1(P.wsc + (size_t)l * P.sc_stride + sc_off_o(P) + r);
    if (threadIdx.x == 0) S.at.t_unit = 0;
    if (have && !S.abort) {
        for (int hoff = 0; hoff < P.G; hoff += GC) attn_unit<DT, GC, KIE_CONS_WARPS>(A, S.at, unit, P.G, hoff);
    }
}

// the two folds of a layer and the down fold's split barrier, by rows per thread
template <int DT, bool F8, int RPT>
__device__ __forceinline__ void o_fold(const KieParams &P, B1Shared &S, uint32_t &ring_it, const uint8_t *ring, int l) {
    float acc[RPT], scl[RPT];
    fold_scales<F8, RPT>(P, l, sc_off_o(P), scl);
    fold_rows<DT, F8, RPT>(P, S, ring_it, ring, PH_OF, acc);
    fold_commit<RPT>(P, S, acc, PH_OF, scl);
}

template <int DT, bool F8, int RPT>
__device__ __forceinline__ void down_fold(const KieParams &P, B1Shared &S, uint32_t &ring_it, const uint8_t *ring,
                                          int l, unsigned long long rd_epoch, int t, int e) {
    float acc[RPT], scl[RPT];
    fold_scales<F8, RPT>(P, l, sc_off_down(P), scl);
    fold_rows<DT, F8, RPT>(P, S, ring_it, ring, PH_DF, acc);
    residual_read_wait(P, S, rd_epoch);  // every CTA has read x for its gate/up norm
    trace_mark(P, t, e + 10);
    fold_commit<RPT>(P, S, acc, PH_DF, scl);
}

// rows per thread of a fold (d <= 4096): 1, 2, 4 or 8
template <int DT, bool F8>
__device__ __forceinline__ void o_fold_any(const KieParams &P, B1Shared &S, uint32_t &ring_it, const uint8_t *ring,
                                           int l) {
    if (P.d <= 512) o_fold<DT, F8, 1>(P, S, ring_it, ring, l);
    else if (P.d <= 1024) o_fold<DT, F8, 2>(P, S, ring_it, ring, l);
    else if (P.d <= 2048) o_fold<DT, F8, 4>(P, S, ring_it, ring, l);
    else o_fold<DT, F8, 8>(P, S, ring_it, ring, l);
}

template <int DT, bool F8>
__device__ __forceinline__ void down_fold_any(const KieParams &P, B1Shared &S, uint32_t &ring_it, const uint8_t *ring,
                                              int l, unsigned long long rd_epoch, int t, int e) {
    if (P.d <= 512) down_fold<DT, F8, 1>(P, S, ring_it, ring, l, rd_epoch, t, e);
    else if (P.d <= 1024) down_fold<DT, F8, 2>(P, S, ring_it, ring, l, rd_epoch, t, e);
    else if (P.d <= 2048) down_fold<DT, F8, 4>(P, S, ring_it, ring, l, rd_epoch, t, e);
    else down_fold<DT, F8, 8>(P, S, ring_it, ring, l, rd_epoch, t, e);
}

// --------------------------------------------------------------- consumer: one command

template <int DT, bool F8>
__device__ void consume(const KieParams &P, B1Shared &S, uint32_t &ring_it, const uint8_t *ring, const KieCmd &cmd,
                        unsigned long long &epoch, unsigned long long &rd_epoch, uint32_t &att_use) {
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
            const float2 sq = gemv_dispatch<DT, F8>(P, S, ring_it, ring, PH_QKV, l, tok, pos, t);
            trace_mark(P, t, e);
            epilogue_qkv<DT>(P, S, l, cmd.sid, pos, tok, sq);
            trace_mark(P, t, e + 1);
            // B: attention, then the O fold
            attention_step<DT, 2>(P, S, l, cmd.sid, pos, epoch, t, e, att_use);  // also serves G == 1
            if (P.trace && t < P.trace_tokens && threadIdx.x == 0)  // end of this CTA's positions (0: no unit)
                P.trace[((size_t)blockIdx.x * P.trace_tokens + t) * P.trace_events + e + 15] = S.at.t_unit;
            trace_mark(P, t, e + 3);
            o_fold_any<DT, F8>(P, S, ring_it, ring, l);
            trace_mark(P, t, e + 4);
            grid_barrier(P, S, epoch, P.timeout_ns, 2);
            trace_mark(P, t, e + 5);
            // C: gate/up, then the down fold
            const float2 sg = gemv_dispatch<DT, F8>(P, S, ring_it, ring, PH_GU, l, tok, pos, t);
            residual_read_arrive(P, S);  // this CTA's reads of x are done
            rd_epoch++;
            trace_mark(P, t, e + 6);
            epilogue_gu(P, S, l, cmd.sid, pos, sg);
            trace_mark(P, t, e + 7);
            down_fold_any<DT, F8>(P, S, ring_it, ring, l, rd_epoch, t, e);
            trace_mark(P, t, e + 8);
            grid_barrier(P, S, epoch, P.timeout_ns, 3);
            trace_mark(P, t, e + 9);
        }
        const int eh = 1 + 16 * L;
        if (head) {
            const float2 sh = gemv_dispatch<DT, F8>(P, S, ring_it, ring, PH_HEAD, L, tok, pos, t);
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
    cp_async_wait_all();  // the L2 reads into warm_sink have landed
}

// --------------------------------------------------------------- the kernel

template <int DT, bool F8>
__global__ void __launch_bounds__(KIE_THREADS, 1) kie_b1_kernel(KieParams P, KieCmd one, int resident) {
    extern __shared__ __align__(1024) uint8_t smem[];
    B1Shared &S = *reinterpret_cast<B1Shared *>(smem + RING_BYTES);
    const int tid = threadIdx.x;
    if (tid == 0) {
        for (int i = 0; i < KIE_NSLOT; i++) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], KIE_CONS_WARPS);  // both groups read every chunk
        }
        fence_mbar_init();
        S.abort = 0;
    }
    if (tid < KIE_NPH) {
        S.row0[tid] = P.row0[tid * (P.nblk + 1) + blockIdx.x];
        S.row1[tid] = P.row0[tid * (P.nblk + 1) + blockIdx.x + 1];
    }
    __syncthreads();
    uint32_t ring_it = 0;  // chunks consumed (consumers) / issued (producer); both advance identically
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
                            P.tokbuf[j] = ((const volatile int32_t *)S.cmd.tokens)[j];
                }
                grid_barrier(P, S, epoch, P.idle_ns + P.timeout_ns, 0);
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
            if (tid == KIE_CONS_THREADS) produce(P, S, ring_it, smem, cmd);
        } else {
            consume<DT, F8>(P, S, ring_it, smem, cmd, epoch, rd_epoch, att_use);
        }
        __syncthreads();
        if (resident && blockIdx.x == 0 && tid == 0) {
            __threadfence_system();
            P.mbox->status = (S.abort || ld_volatile_u32(P.err) != 0u) ? -1 : 0;
            st_release_sys_u32(&P.mbox->done_seq, cmd.seq);
        }
        if (!resident || S.abort) break;
    }
}

}  // namespace

// --------------------------------------------------------------- host-side launch helpers

extern "C++" {

size_t kie_b1_smem_bytes() { return RING_BYTES + sizeof(B1Shared); }

// rows per ring chunk for row length K, and the most rows one CTA may own in such a phase
int kie_b1_chunk_rows(int K) { return (KIE_CONS_WARPS / col_slices(K)) * rows_per_group(K); }
int kie_b1_max_rows(int K) { return WPART_FLOATS / col_slices(K); }

// the kernel instantiation for a storage dtype and weight format
static const void *b1_fn(int dtype, bool f8) {
    if (dtype == KIE_BF16) return f8 ? (const void *)kie_b1_kernel<KIE_BF16, true> : (const void *)kie_b1_kernel<KIE_BF16, false>;
    return f8 ? (const void *)kie_b1_kernel<KIE_FP16, true> : (const void *)kie_b1_kernel<KIE_FP16, false>;
}

cudaError_t kie_b1_prepare(int dtype, bool f8) {
    return cudaFuncSetAttribute(b1_fn(dtype, f8), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kie_b1_smem_bytes());
}

cudaError_t kie_b1_occupancy(int dtype, bool f8, int *blocks_per_sm) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, b1_fn(dtype, f8), KIE_THREADS, kie_b1_smem_bytes());
}

cudaError_t kie_b1_launch(const KieParams &P, const KieCmd &one, int resident, cudaStream_t stream) {
    // the attention merge counters count up from zero within a launch
    const cudaError_t e = cudaMemsetAsync(P.cnt, 0, (size_t)P.Hkv * sizeof(unsigned), stream);
    if (e != cudaSuccess) return e;
    KieParams p = P;
    KieCmd c = one;
    int r = resident;
    void *args[] = {&p, &c, &r};
    return cudaLaunchCooperativeKernel(b1_fn(P.dtype, P.wesz == 1), dim3(P.nblk), dim3(KIE_THREADS), args,
                                       kie_b1_smem_bytes(), stream);
}

}  // extern "C++"
