// Split-K single-query attention over an fp16/bf16 KV cache (one decode position).
//
// Decode reads the whole KV cache once per token ("Kog 3000 tok/s 实时推理…", section
// 内存带宽优化的三层策略), so the cache range of each kv head is cut into `nsplit` splits
// and one CTA works on one (kv head, split) unit, for all query heads of the group.
//
// Within a unit, D/8 lanes hold one position's 16-byte slices ("a position group"), so a
// warp covers 32/(D/8) positions per load and the CTA 8x that. Each position group walks
// its positions in batches of B, issuing all 2B K/V loads of a batch before using any, and
// keeps a running softmax per query head (max m, sum l, weighted value sum acc), with
// scores in log2 units: s_j = q . K_j * log2(e) / sqrt(D), p_j = 2^(s_j - m).
// Position groups, then warps, are merged by rescaling to the common max. The last unit to
// finish a kv head combines the splits the same way:
//     o = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s,
// which equals the one-pass softmax over all positions for any split count (the merge
// issues each step's loads together, so it costs two L2 round trips for any split count).
//
// Contract for callers: NW warps (8 or 16, threads 0 .. 32*NW-1) execute attn_all_units
// together and use named barrier 1.
#pragma once
#include <math_constants.h>

#include "kie_device.cuh"

struct AttnArgs {
    const float *q;          // [Hq][D] fp32 (already rotated)
    const uint16_t *k, *v;   // kv head 0, position 0 of the cache
    long long head_stride;   // elements between consecutive kv heads
    float *part;             // [Hkv * nsplit * G][D + 2] partials (m, l, acc)
    unsigned *cnt;           // [Hkv] finished-split counters (0 on entry, left at 0)
    float *o;                // [Hq][D] output (unused when bpack is set)
    uint8_t *bpack;          // or null: the output goes, as 16-bit hi/lo halves, to row brow
                             // (hi) and 64 + brow (lo) of the swizzled 128 x 64 tiles of the
                             // tick kernel's B operand (column h * D + e)
    int brow;
    int gout;                // kv head whose output columns a unit writes; -1: unit / nsplit
    uint32_t cnt_target;     // 0: the last split merges. Else every split merges a slice of its kv
                             // head's output once cnt[kv head] reaches this value (the counters
                             // then only count up): elements [8 q0, 8 q1) of the kv head's Gt * D
                             // outputs, q0 = s * (Gt * D / 8) / nsplit (8-element groups), written
                             // to oslice[0 .. 8 (q1 - q0)) (shared memory)
    float *oslice;
    long long timeout_ns;    // bound of that wait; on expiry err gets an error code
    unsigned *err;
    int D, Hkv, nsplit, ctx;
};

struct AttnSmem {
    float wacc[4][KIE_GMAX * KIE_DMAX];  // warp w adds into slot w % 4, in warp order
    float wl[4][KIE_GMAX];
    float mrow[KIE_GMAX];
    float red[KIE_GMAX * 16];
    int is_last;
    uint32_t pub_sink;          // scratch word of pub_wait
    unsigned long long t_unit;  // globaltimer when this CTA's last unit finished its positions
};

// Asks L2 for the K and V rows units first, first + step, ... will read (a hint that may be
// issued before the newest position is written: L2 stays coherent).
KIE_DEV void attn_prefetch(const uint16_t *k, const uint16_t *v, long long head_stride, int D, int Hkv, int nsplit,
                           int ctx, int first, int step) {
    for (int unit = first; unit < Hkv * nsplit; unit += step) {
        const int g = unit / nsplit, s = unit % nsplit;
        const long long p0 = (long long)s * ctx / nsplit, p1 = (long long)(s + 1) * ctx / nsplit;
        for (long long a = p0; a < p1; a += 1024) {
            const long long n = (p1 - a < 1024 ? p1 - a : 1024) * D * 2;
            const size_t off = (size_t)g * head_stride + (size_t)a * D;
            bulk_prefetch_l2(k + off, (uint32_t)n);
            bulk_prefetch_l2(v + off, (uint32_t)n);
        }
    }
}

// positions per position group per batch (register budget)
template <int GC, int NW>
__host__ __device__ constexpr int attn_batch() {
    return NW >= 16 ? (GC == 1 ? 4 : 2) : (GC == 1 ? 8 : GC == 2 ? 4 : 2);
}

// 2^(x - M) with 2^(-inf - M) = 0 (M >= x; M = -inf only when x = -inf)
KIE_DEV float rescale(float x, float M) { return x == -CUDART_INF_F ? 0.f : exp2f(x - M); }

// One batch of a position group: the scores of its B positions base + gi + b * ngroups
// (those >= np count as -inf) for the G query heads, then the running softmax update of
// (m, l, acc); the D/8 lanes of a position hold 16-byte slices of its K and V rows.
template <int DT, int G, int B>
KIE_DEV void attn_update(const uint4 (&kv)[B], const uint4 (&vv)[B], int base, int np, int gi, int ngroups, int lpp,
                         const float (&q)[G][8], float (&m)[G], float (&l)[G], float (&acc)[G][8]) {
    float sc[B][G];
#pragma unroll
    for (int b = 0; b < B; b++) {
        const bool ok = base + gi + b * ngroups < np;
        float f[8];
        cvt8<DT>(kv[b], f);
#pragma unroll
        for (int jj = 0; jj < G; jj++) {
            float d = 0.f;
#pragma unroll
            for (int e = 0; e < 8; e++) d = fmaf(f[e], q[jj][e], d);
            for (int o = lpp >> 1; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            sc[b][jj] = ok ? d : -CUDART_INF_F;
        }
    }
#pragma unroll
    for (int jj = 0; jj < G; jj++) {
        float mb = m[jj];
#pragma unroll
        for (int b = 0; b < B; b++) mb = fmaxf(mb, sc[b][jj]);
        const float r = rescale(m[jj], mb);
        l[jj] *= r;
#pragma unroll
        for (int e = 0; e < 8; e++) acc[jj][e] *= r;
        m[jj] = mb;
    }
#pragma unroll
    for (int b = 0; b < B; b++) {
        float f[8];
        cvt8<DT>(vv[b], f);
#pragma unroll
        for (int jj = 0; jj < G; jj++) {
            const float p = rescale(sc[b][jj], m[jj]);
            l[jj] += p;
#pragma unroll
            for (int e = 0; e < 8; e++) acc[jj][e] = fmaf(p, f[e], acc[jj][e]);
        }
    }
}

// output elements col, col + 1 (col even): fp32 to A.o, or hi/lo 16-bit halves into the packed
// B operand of the tick kernel
template <int DT>
KIE_DEV void attn_out2(const AttnArgs &A, int col, float o0, float o1) {
    if (A.bpack) {
        uint8_t *tile = A.bpack + (size_t)(col >> 6) * 16384;
        const uint32_t within = (uint32_t)(col & 7) * 2;
        const uint16_t h0 = store1<DT>(o0), h1 = store1<DT>(o1);
        const uint16_t l0 = store1<DT>(o0 - cvt1<DT>(h0)), l1 = store1<DT>(o1 - cvt1<DT>(h1));
        *reinterpret_cast<uint32_t *>(tile + sw128(A.brow, (col >> 3) & 7) + within) = (uint32_t)h0 | ((uint32_t)h1 << 16);
        *reinterpret_cast<uint32_t *>(tile + sw128(64 + A.brow, (col >> 3) & 7) + within) = (uint32_t)l0 | ((uint32_t)l1 << 16);
    } else {
        *reinterpret_cast<float2 *>(A.o + col) = make_float2(o0, o1);
    }
}

template <int DT, int GC, int NW, bool DIRECT>
__device__ __forceinline__ void attn_tail(const AttnArgs &A, AttnSmem &S, int unit, int Gt, int hoff, float (&m)[GC], float (&l)[GC],
                          float (&acc)[GC][8]);

template <int DT, int GC, int NW>
__device__ void attn_unit(const AttnArgs &A, AttnSmem &S, int unit, int Gt, int hoff) {
    constexpr int G = GC;
    constexpr int B = attn_batch<GC, NW>();
    constexpr int ATTN_WARPS = NW, ATTN_THREADS = NW * 32;
    const int nh = min(GC, Gt - hoff);
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int D = A.D, lpp = D >> 3, ppw = 32 / lpp, sub = lane / lpp, sl = lane % lpp;
    const int nsplit = A.nsplit, ctx = A.ctx;
    const int ngroups = ATTN_WARPS * ppw, gi = w * ppw + sub;
    const float qscale = rsqrtf((float)D) * 1.4426950408889634f;

    const int g = unit / nsplit, s = unit % nsplit;
    const int p0 = (int)((long long)s * ctx / nsplit), p1 = (int)((long long)(s + 1) * ctx / nsplit);
    const int np = p1 - p0;
    const size_t kvoff = (size_t)g * A.head_stride + (size_t)p0 * D + sl * 8;
    const uint16_t *Kp = A.k + kvoff;
    const uint16_t *Vp = A.v + kvoff;

    float q[G][8];
#pragma unroll
    for (int jj = 0; jj < G; jj++) {
        const float *qp = A.q + (size_t)(g * Gt + hoff + min(jj, nh - 1)) * D + sl * 8;
        const float4 a = __ldcg(reinterpret_cast<const float4 *>(qp));
        const float4 b = __ldcg(reinterpret_cast<const float4 *>(qp + 4));
        q[jj][0] = a.x * qscale; q[jj][1] = a.y * qscale; q[jj][2] = a.z * qscale; q[jj][3] = a.w * qscale;
        q[jj][4] = b.x * qscale; q[jj][5] = b.y * qscale; q[jj][6] = b.z * qscale; q[jj][7] = b.w * qscale;
    }
    float m[G], l[G], acc[G][8];
#pragma unroll
    for (int jj = 0; jj < G; jj++) {
        m[jj] = -CUDART_INF_F;
        l[jj] = 0.f;
#pragma unroll
        for (int e = 0; e < 8; e++) acc[jj][e] = 0.f;
    }

    auto batch = [&](int base, const uint4 (&kv)[B], const uint4 (&vv)[B]) {
        attn_update<DT, G, B>(kv, vv, base, np, gi, ngroups, lpp, q, m, l, acc);
    };
    for (int base = 0; base < np; base += ngroups * B) {  // uniform across the CTA
        uint4 kv[B], vv[B];
#pragma unroll
        for (int b = 0; b < B; b++) {
            const int j = base + gi + b * ngroups;
            const bool ok = j < np;
            kv[b] = ok ? __ldcg(reinterpret_cast<const uint4 *>(Kp + (size_t)j * D)) : make_uint4(0, 0, 0, 0);
            vv[b] = ok ? __ldcg(reinterpret_cast<const uint4 *>(Vp + (size_t)j * D)) : make_uint4(0, 0, 0, 0);
        }
        batch(base, kv, vv);
    }
    attn_tail<DT, GC, NW, (NW < 16)>(A, S, unit, Gt, hoff, m, l, acc);
}

// The end of a unit: merge the position groups and warps of this CTA at their common max;
// with one split the result is final (o = acc / l: written directly when DIRECT), otherwise
// publish the split's partial and let the last split of the kv head merge all of them.
// (The 16-warp batch-1 kernel, whose units always have several splits at its sizes, leaves
// DIRECT out to keep registers for its main loop; the general merge is exact for one split.)
template <int DT, int GC, int NW, bool DIRECT>
__device__ __forceinline__ void attn_tail(const AttnArgs &A, AttnSmem &S, int unit, int Gt, int hoff, float (&m)[GC], float (&l)[GC],
                          float (&acc)[GC][8]) {
    constexpr int G = GC;
    constexpr int ATTN_WARPS = NW, ATTN_THREADS = NW * 32;
    const int nh = min(GC, Gt - hoff);
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int D = A.D, lpp = D >> 3, sub = lane / lpp, sl = lane % lpp;
    const int nsplit = A.nsplit;
    const int g = unit / nsplit;
    const int go = A.gout >= 0 ? A.gout : g;  // the kv head of the output columns
    // merge the position groups of each warp (lanes with the same sl hold the same dims)
#pragma unroll
    for (int jj = 0; jj < G; jj++) {
        for (int o = lpp; o < 32; o <<= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m[jj], o);
            const float l2 = __shfl_xor_sync(0xffffffffu, l[jj], o);
            const float M = fmaxf(m[jj], m2);
            const float ra = rescale(m[jj], M), rb = rescale(m2, M);
            l[jj] = l[jj] * ra + l2 * rb;
#pragma unroll
            for (int e = 0; e < 8; e++) {
                const float a2 = __shfl_xor_sync(0xffffffffu, acc[jj][e], o);
                acc[jj][e] = acc[jj][e] * ra + a2 * rb;
            }
            m[jj] = M;
        }
        if (lane == 0) S.red[w * G + jj] = m[jj];
    }
    named_bar_sync(1, ATTN_THREADS);
    if (tid < G) {
        float M = -CUDART_INF_F;
        for (int k = 0; k < ATTN_WARPS; k++) M = fmaxf(M, S.red[k * G + tid]);
        S.mrow[tid] = M;
    }
    named_bar_sync(1, ATTN_THREADS);
    // merge the warps at the common max, in a fixed order (warps w, w+4, ... into slot w % 4,
    // then slots 0..3)
    for (int round = 0; round < ATTN_WARPS / 4; round++) {
        if ((w >> 2) == round && sub == 0) {
            float *wa = S.wacc[w & 3];
#pragma unroll
            for (int jj = 0; jj < G; jj++) {
                const float r = rescale(m[jj], S.mrow[jj]);
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    const float v = acc[jj][e] * r;
                    wa[jj * D + sl * 8 + e] = round == 0 ? v : wa[jj * D + sl * 8 + e] + v;
                }
                if (sl == 0) S.wl[w & 3][jj] = round == 0 ? l[jj] * r : S.wl[w & 3][jj] + l[jj] * r;
            }
        }
        named_bar_sync(1, ATTN_THREADS);
    }

    if (tid == 0) S.t_unit = globaltimer();
    if (DIRECT && nsplit == 1) {  // the only split: o = acc / l
        for (int i = tid; i < nh * D / 2; i += ATTN_THREADS) {
            const int jj = (2 * i) / D, e = (2 * i) % D, k = jj * D + e;
            const float den = ((S.wl[0][jj] + S.wl[1][jj]) + S.wl[2][jj]) + S.wl[3][jj];
            const float n0 = ((S.wacc[0][k] + S.wacc[1][k]) + S.wacc[2][k]) + S.wacc[3][k];
            const float n1 = ((S.wacc[0][k + 1] + S.wacc[1][k + 1]) + S.wacc[2][k + 1]) + S.wacc[3][k + 1];
            attn_out2<DT>(A, (go * Gt + hoff + jj) * D + e, n0 / den, n1 / den);
        }
        named_bar_sync(1, ATTN_THREADS);
        return;
    }
    // publish this split's partial, then the last split of the kv head merges. With cnt_target
    // (the batch-1 megakernel, whose weight stream keeps bulk copies in flight) the partial is
    // published by completion and the split's count is a relaxed add; else by a fence.
    float *pp = A.part + ((size_t)unit * Gt + hoff) * (D + 2);
    uint32_t ptok = 0;
    for (int i = tid; i < nh * (D + 2) / 2; i += ATTN_THREADS) {  // float2 per thread (D + 2 is even)
        const int jj = (2 * i) / (D + 2), e = (2 * i) % (D + 2);
        float2 val;
        if (e == 0) {
            val.x = S.mrow[jj];
            val.y = ((S.wl[0][jj] + S.wl[1][jj]) + S.wl[2][jj]) + S.wl[3][jj];
        } else {
            const int k = jj * D + e - 2;
            val.x = ((S.wacc[0][k] + S.wacc[1][k]) + S.wacc[2][k]) + S.wacc[3][k];
            val.y = ((S.wacc[0][k + 1] + S.wacc[1][k + 1]) + S.wacc[2][k + 1]) + S.wacc[3][k + 1];
        }
        if (!in_bounds(((size_t)unit * Gt + hoff) * (D + 2) + 2 * i + 1 < (size_t)A.Hkv * nsplit * Gt * (D + 2), A.err, 0x30))
            continue;
        if (A.cnt_target) pub_f32x2(pp + 2 * i, val.x, val.y, ptok);
        else reinterpret_cast<float2 *>(pp)[i] = val;
    }
    if (A.cnt_target) pub_wait(ptok, &S.pub_sink);
    else __threadfence();
    named_bar_sync(1, ATTN_THREADS);
    if (A.cnt_target) {
        // Every split merges its own slice of the kv head's output once all splits have
        // published (after its last pass over the query heads): one (m, l) + partial-sum load
        // for all splits, in a single round trip, and no single CTA merging everything.
        const bool last_pass = hoff + GC >= Gt;
        if (tid == 0) {
            red_relaxed_gpu_add_u32(A.cnt + g, 1u);
            const uint64_t t0 = globaltimer();
            unsigned spins = 0;
            while (last_pass && (int)(ld_acquire_gpu_u32(A.cnt + g) - A.cnt_target) < 0) {
                if ((++spins & 63u) == 0) {
                    if (ld_volatile_u32(A.err) != 0u) break;  // another CTA failed: give up
                    if ((long long)(globaltimer() - t0) > A.timeout_ns) {
                        set_error(A.err, DERR_BARRIER_TIMEOUT, 0x50);
                        break;
                    }
                }
            }
        }
        named_bar_sync(1, ATTN_THREADS);
        if (!last_pass) return;
        const int s = unit % nsplit, E = Gt * D, nq = E / 8;
        const int e0 = 8 * (int)((long long)s * nq / nsplit), e1 = 8 * (int)((long long)(s + 1) * nq / nsplit);
        const int ne = e1 - e0;
        if (ne == 0) return;  // more splits than 8-element groups: this split owns no slice
        const float *pg = A.part + (size_t)g * nsplit * Gt * (D + 2);
        float *ek = &S.wacc[0][0];   // [nsplit][Gt] max, then weights
        float *lk = ek + nsplit * Gt;  // [nsplit][Gt] sums
        float *ak = lk + nsplit * Gt;  // [nsplit][ne] partial sums of this slice
        for (int i = tid; i < nsplit * Gt + nsplit * ne; i += ATTN_THREADS) {
            if (i < nsplit * Gt) {
                const float2 ml = __ldcg(reinterpret_cast<const float2 *>(pg + (size_t)i * (D + 2)));
                ek[i] = ml.x;
                lk[i] = ml.y;
            } else {
                const int j = i - nsplit * Gt, k = j / ne, ee = e0 + j % ne;
                ak[j] = __ldcg(pg + ((size_t)k * Gt + ee / D) * (D + 2) + 2 + ee % D);
            }
        }
        named_bar_sync(1, ATTN_THREADS);
        if (tid < Gt) {
            float M = -CUDART_INF_F;
            for (int k = 0; k < nsplit; k++) M = fmaxf(M, ek[k * Gt + tid]);
            float den = 0.f;
            for (int k = 0; k < nsplit; k++) {
                const float e = rescale(ek[k * Gt + tid], M);
                ek[k * Gt + tid] = e;
                den = fmaf(e, lk[k * Gt + tid], den);
            }
            S.red[tid] = den;
        }
        named_bar_sync(1, ATTN_THREADS);
        for (int j = tid; j < ne; j += ATTN_THREADS) {  // splits added in ascending order
            const int ee = e0 + j, jj = ee / D;
            float num = 0.f;
            for (int k = 0; k < nsplit; k++) num = fmaf(ek[k * Gt + jj], ak[k * ne + j], num);
            A.oslice[j] = num / S.red[jj];
        }
        named_bar_sync(1, ATTN_THREADS);
        return;
    }
    if (tid == 0) {
        const unsigned chunks = (unsigned)((Gt + GC - 1) / GC);
        const unsigned prev = atomicAdd(A.cnt + g, 1u);
        S.is_last = (prev == (unsigned)nsplit * chunks - 1u);
    }
    named_bar_sync(1, ATTN_THREADS);
    if (S.is_last) {
        __threadfence();
        // All loads of a step are issued before any is used, so the merge costs two L2
        // round trips whatever the split count: (1) every split's (m, l); (2) per query head
        // M = max m_k, e_k = 2^(m_k - M) and den = sum e_k l_k; (3) per output pair
        // num = sum e_k acc_k, the splits shared out over TPP adjacent lanes (each adds its
        // splits in ascending order, then a fixed shuffle tree), o = num / den.
        const float *pg = A.part + (size_t)g * nsplit * Gt * (D + 2);
        float *ek = &S.wacc[0][0];  // [nsplit][Gt] (the warp sums were published above)
        float *lk = ek + nsplit * Gt;
        for (int i = tid; i < nsplit * Gt; i += ATTN_THREADS) {
            const float2 ml = __ldcg(reinterpret_cast<const float2 *>(pg + (size_t)i * (D + 2)));
            ek[i] = ml.x;
            lk[i] = ml.y;
        }
        named_bar_sync(1, ATTN_THREADS);
        if (tid < Gt) {
            float M = -CUDART_INF_F;
            for (int k = 0; k < nsplit; k++) M = fmaxf(M, ek[k * Gt + tid]);
            float den = 0.f;
            for (int k = 0; k < nsplit; k++) {
                const float e = rescale(ek[k * Gt + tid], M);
                ek[k * Gt + tid] = e;
                den = fmaf(e, lk[k * Gt + tid], den);
            }
            S.red[tid] = den;
        }
        named_bar_sync(1, ATTN_THREADS);
        const int npairs = Gt * D / 2;
        int tpp = 1;  // lanes per output pair: a power of two <= 16
        while (tpp < 16 && tpp * 2 * npairs <= ATTN_THREADS) tpp <<= 1;
        for (int i0 = 0; i0 < npairs * tpp; i0 += ATTN_THREADS) {  // uniform across the CTA
            const int i = i0 + tid, pr = i / tpp, sub = i % tpp;
            float2 num = make_float2(0.f, 0.f);
            const int jj = (2 * pr) / D, e = (2 * pr) % D;
            if (pr < npairs) {
                const float *pe = pg + (size_t)jj * (D + 2) + 2 + e;
                constexpr int MU = NW >= 16 ? 8 : 4;  // loads in flight per lane (register budget)
                for (int kb = sub; kb < nsplit; kb += MU * tpp) {
                    float2 v[MU];
                    float wk[MU];
#pragma unroll
                    for (int u = 0; u < MU; u++) {
                        const int k = kb + u * tpp;
                        const bool ok = k < nsplit;
                        v[u] = ok ? __ldcg(reinterpret_cast<const float2 *>(pe + (size_t)k * Gt * (D + 2)))
                                  : make_float2(0.f, 0.f);
                        wk[u] = ok ? ek[k * Gt + jj] : 0.f;
                    }
#pragma unroll
                    for (int u = 0; u < MU; u++) {
                        num.x = fmaf(wk[u], v[u].x, num.x);
                        num.y = fmaf(wk[u], v[u].y, num.y);
                    }
                }
            }
            for (int o = 1; o < tpp; o <<= 1) {
                num.x += __shfl_xor_sync(0xffffffffu, num.x, o);
                num.y += __shfl_xor_sync(0xffffffffu, num.y, o);
            }
            if (pr < npairs && sub == 0) {
                const float den = S.red[jj];
                attn_out2<DT>(A, (go * Gt + jj) * D + e, num.x / den, num.y / den);
            }
        }
        if (tid == 0) A.cnt[g] = 0u;
    }
    named_bar_sync(1, ATTN_THREADS);
}

// Units first, first + step, ... of the Hkv * nsplit units. With 16 warps (a smaller
// register budget per thread) at most 2 query heads are processed per pass, else 4.
template <int DT, int NW>
__device__ void attn_all_units(const AttnArgs &A, AttnSmem &S, int G, int first, int step) {
    constexpr int GCMAX = NW >= 16 ? 2 : 4;
    for (int unit = first; unit < A.Hkv * A.nsplit; unit += step) {
        if (G == 1) {
            attn_unit<DT, 1, NW>(A, S, unit, 1, 0);
        } else if (G <= GCMAX) {
            if (G == 2) attn_unit<DT, 2, NW>(A, S, unit, 2, 0);
            else if (G == 3) attn_unit<DT, (GCMAX >= 3 ? 3 : 2), NW>(A, S, unit, 3, 0);
            else attn_unit<DT, GCMAX, NW>(A, S, unit, G, 0);
        } else {
            for (int hoff = 0; hoff < G; hoff += GCMAX) attn_unit<DT, GCMAX, NW>(A, S, unit, G, hoff);
        }
    }
}
