// Split-K single-query attention over an fp16/bf16 KV cache (one decode position).
//
// Decode reads the whole KV cache once per token ("Kog 3000 tok/s 实时推理…", section
// 内存带宽优化的三层策略), so the cache range of each kv head is cut into `nsplit` splits
// and one CTA works on one (kv head, split) unit, for all query heads of the group:
//
//   pass 1  s_j = q_h . K_j / sqrt(D) (kept in log2 units) for every position of the split
//   pass 2  p_j = 2^(s_j - m), l = sum p_j, acc = sum p_j V_j
//   merge   the last unit to finish a kv head combines the splits' (m, l, acc):
//           o = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s
//
// The merge is the usual log-sum-exp combination of partial softmaxes (it equals the
// one-pass softmax for any number of splits). Lanes: D/8 lanes hold one position's
// 16-byte slices, so a warp covers 32/(D/8) positions per load; the partial sums over
// positions in a warp are combined with shuffles, across warps in shared memory.
//
// Contract for callers: 256 threads (8 warps) execute attn_all_units together and use
// named barrier 1; AttnSmem is zero-initialised once with attn_smem_init.
#pragma once
#include <math_constants.h>

#include "kie_device.cuh"

struct AttnArgs {
    const float *q;          // [Hq][D] fp32 (already rotated)
    const uint16_t *k, *v;   // kv head 0, position 0 of the cache
    long long head_stride;   // elements between consecutive kv heads
    float *part;             // [Hkv * nsplit * G][D + 2] partials (m, l, acc)
    unsigned *cnt;           // [Hkv] finished-split counters (0 on entry, left at 0)
    float *o;                // [Hq][D] output
    int D, Hkv, nsplit, ctx;
};

struct AttnSmem {
    float scores[KIE_SCORE_MAX];
    float accs[KIE_GMAX * KIE_DMAX];
    float lsum[KIE_GMAX];
    float mrow[KIE_GMAX];
    float red[KIE_GMAX * 8];
    int is_last;
};

KIE_DEV void attn_smem_init(AttnSmem &S, int tid, int nthreads) {
    for (int i = tid; i < KIE_GMAX * KIE_DMAX; i += nthreads) S.accs[i] = 0.f;
    if (tid < KIE_GMAX) S.lsum[tid] = 0.f;
}

#define ATTN_THREADS 256
#define ATTN_WARPS 8

template <int DT, int G>
__device__ void attn_unit(const AttnArgs &A, AttnSmem &S, int unit) {
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int D = A.D, lpp = D >> 3, ppw = 32 / lpp, sub = lane / lpp, sl = lane % lpp;
    const int nsplit = A.nsplit, ctx = A.ctx;
    const int SP = KIE_SCORE_MAX / G;
    const float qscale = rsqrtf((float)D) * 1.4426950408889634f;
    const int stride = ATTN_WARPS * ppw;
    constexpr int U = 4;

    const int g = unit / nsplit, s = unit % nsplit;
    const int p0 = (int)((long long)s * ctx / nsplit), p1 = (int)((long long)(s + 1) * ctx / nsplit);
    const int np = p1 - p0;
    const size_t kvoff = (size_t)g * A.head_stride + (size_t)p0 * D + sl * 8;
    const uint16_t *Kp = A.k + kvoff;
    const uint16_t *Vp = A.v + kvoff;

    float q[G][8];
#pragma unroll
    for (int jj = 0; jj < G; jj++) {
        const float *qp = A.q + (size_t)(g * G + jj) * D + sl * 8;
        const float4 a = __ldcg(reinterpret_cast<const float4 *>(qp));
        const float4 b = __ldcg(reinterpret_cast<const float4 *>(qp + 4));
        q[jj][0] = a.x * qscale; q[jj][1] = a.y * qscale; q[jj][2] = a.z * qscale; q[jj][3] = a.w * qscale;
        q[jj][4] = b.x * qscale; q[jj][5] = b.y * qscale; q[jj][6] = b.z * qscale; q[jj][7] = b.w * qscale;
    }

    // pass 1: scores of every position of the split
    float mx[G];
#pragma unroll
    for (int jj = 0; jj < G; jj++) mx[jj] = -CUDART_INF_F;
    for (int j0 = w * ppw + sub; j0 - sub < np; j0 += stride * U) {
        uint4 kv[U];
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int j = j0 + u * stride;
            kv[u] = j < np ? __ldcg(reinterpret_cast<const uint4 *>(Kp + (size_t)j * D)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int j = j0 + u * stride;
            float f[8];
            cvt8<DT>(kv[u], f);
#pragma unroll
            for (int jj = 0; jj < G; jj++) {
                float dsum = 0.f;
#pragma unroll
                for (int e = 0; e < 8; e++) dsum = fmaf(f[e], q[jj][e], dsum);
                for (int o = lpp >> 1; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
                if (j < np) {
                    if (sl == 0) S.scores[jj * SP + j] = dsum;
                    mx[jj] = fmaxf(mx[jj], dsum);
                }
            }
        }
    }
#pragma unroll
    for (int jj = 0; jj < G; jj++) {
        const float m = warp_max(mx[jj]);
        if (lane == 0) S.red[w * G + jj] = m;
    }
    named_bar_sync(1, ATTN_THREADS);
    if (tid < G) {
        float m = -CUDART_INF_F;
        for (int k = 0; k < ATTN_WARPS; k++) m = fmaxf(m, S.red[k * G + tid]);
        S.mrow[tid] = m;
    }
    named_bar_sync(1, ATTN_THREADS);
    float M[G];
#pragma unroll
    for (int jj = 0; jj < G; jj++) M[jj] = S.mrow[jj];

    // pass 2: softmax weights and the weighted sum of values
    float acc[G][8], ls[G];
#pragma unroll
    for (int jj = 0; jj < G; jj++) {
        ls[jj] = 0.f;
#pragma unroll
        for (int e = 0; e < 8; e++) acc[jj][e] = 0.f;
    }
    for (int j0 = w * ppw + sub; j0 - sub < np; j0 += stride * U) {
        uint4 vv[U];
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int j = j0 + u * stride;
            vv[u] = j < np ? __ldcg(reinterpret_cast<const uint4 *>(Vp + (size_t)j * D)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int j = j0 + u * stride;
            if (j < np) {
                float f[8];
                cvt8<DT>(vv[u], f);
#pragma unroll
                for (int jj = 0; jj < G; jj++) {
                    const float p = exp2f(S.scores[jj * SP + j] - M[jj]);
                    ls[jj] += p;
#pragma unroll
                    for (int e = 0; e < 8; e++) acc[jj][e] = fmaf(p, f[e], acc[jj][e]);
                }
            }
        }
    }
#pragma unroll
    for (int jj = 0; jj < G; jj++) {
        for (int o = lpp; o < 32; o <<= 1) {
            ls[jj] += __shfl_xor_sync(0xffffffffu, ls[jj], o);
#pragma unroll
            for (int e = 0; e < 8; e++) acc[jj][e] += __shfl_xor_sync(0xffffffffu, acc[jj][e], o);
        }
        if (sub == 0) {
#pragma unroll
            for (int e = 0; e < 8; e++) atomicAdd(&S.accs[jj * D + sl * 8 + e], acc[jj][e]);
            if (sl == 0) atomicAdd(&S.lsum[jj], ls[jj]);
        }
    }
    named_bar_sync(1, ATTN_THREADS);

    // publish this split's partial, then the last split of the kv head merges
    float *pp = A.part + (size_t)unit * G * (D + 2);
    for (int i = tid; i < G * (D + 2); i += ATTN_THREADS) {
        const int jj = i / (D + 2), e = i % (D + 2);
        float val;
        if (e == 0) {
            val = M[jj];
        } else if (e == 1) {
            val = S.lsum[jj];
            S.lsum[jj] = 0.f;
        } else {
            val = S.accs[jj * D + e - 2];
            S.accs[jj * D + e - 2] = 0.f;
        }
        pp[i] = val;
    }
    __threadfence();
    named_bar_sync(1, ATTN_THREADS);
    if (tid == 0) {
        const unsigned prev = atomicAdd(A.cnt + g, 1u);
        S.is_last = (prev == (unsigned)(nsplit - 1));
    }
    named_bar_sync(1, ATTN_THREADS);
    if (S.is_last) {
        __threadfence();
        const float *pg = A.part + (size_t)g * nsplit * G * (D + 2);
        for (int i = tid; i < G * D; i += ATTN_THREADS) {
            const int jj = i / D, e = i % D;
            float mxs = -CUDART_INF_F;
            for (int k = 0; k < nsplit; k++) mxs = fmaxf(mxs, __ldcg(pg + ((size_t)k * G + jj) * (D + 2)));
            float num = 0.f, den = 0.f;
            for (int k = 0; k < nsplit; k++) {
                const float *pk = pg + ((size_t)k * G + jj) * (D + 2);
                const float wk = exp2f(__ldcg(pk) - mxs);
                den = fmaf(wk, __ldcg(pk + 1), den);
                num = fmaf(wk, __ldcg(pk + 2 + e), num);
            }
            A.o[(size_t)(g * G + jj) * D + e] = num / den;
        }
        if (tid == 0) A.cnt[g] = 0u;
    }
    named_bar_sync(1, ATTN_THREADS);
}

// Units first, first + step, ... of the Hkv * nsplit units.
template <int DT>
__device__ void attn_all_units(const AttnArgs &A, AttnSmem &S, int G, int first, int step) {
    for (int unit = first; unit < A.Hkv * A.nsplit; unit += step) {
        switch (G) {
            case 1: attn_unit<DT, 1>(A, S, unit); break;
            case 2: attn_unit<DT, 2>(A, S, unit); break;
            case 3: attn_unit<DT, 3>(A, S, unit); break;
            case 4: attn_unit<DT, 4>(A, S, unit); break;
            case 5: attn_unit<DT, 5>(A, S, unit); break;
            case 6: attn_unit<DT, 6>(A, S, unit); break;
            case 7: attn_unit<DT, 7>(A, S, unit); break;
            default: attn_unit<DT, 8>(A, S, unit); break;
        }
    }
}
