// Batch-1 decode megakernel for sm_100a.
//
// One CTA per SM stays resident across layers and tokens (the persistent single-kernel
// runtime of the HN digest of Kog's inference engine, section 技术原理, and the resident GPU
// program of "实时AI推理为何贵56倍？…", section 让工作常驻 GPU). A decode step streams every weight
// byte plus the KV cache once ("Kog 3000 tok/s 实时推理…", section 内存带宽优化的三层策略), so
// the kernel is organised around that stream:
//
//  * Warp 8 (the producer) walks this CTA's fixed weight schedule for the whole command
//    (all layers, all tokens) and copies it, chunk by chunk, into a 6 x 32 KB shared-memory
//    ring with 1-D bulk async copies (TMA). The schedule is contiguous in HBM because the
//    weights were repacked at engine creation in exactly this order, so each SM streams one
//    disjoint span (the aligned, topology-aware access pattern of the same section). The
//    producer never waits on grid barriers, so weight streaming runs ahead of compute by up
//    to the ring size across phase, layer and token boundaries.
//  * Warps 0-7 (consumers) run the phases of each layer on the staged chunks:
//      QKV  : RMSNorm -> [Wq;Wk;Wv] rows -> RoPE -> q, and the K/V append to the cache
//      ATTN : split-K single-query attention over the cache, last split merges (LSE)
//      O    : x += Wo o
//      GU   : RMSNorm -> gate/up rows -> u = silu(gate) * up
//      DOWN : x += Wd u
//    then, per token, HEAD: final RMSNorm -> LM-head rows -> block argmax -> grid argmax.
//    Phases are separated by a grid-wide barrier with a time limit.
//
// GEMV mapping: a ring chunk holds CR whole rows of length K. Warp w owns the column slice
// [w*K/8, (w+1)*K/8); lane l owns 16-byte vectors l, l+32, ... of that slice, so a lane's
// slice of the input vector sits in registers for the whole phase and each staged weight
// byte is read from shared memory exactly once. Row sums are reduced across the warp
// (shuffle butterfly over CR rows) and across warps with shared-memory atomics.
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kie_attn.cuh"
#include "kie_device.cuh"

namespace {

constexpr int RING_BYTES = KIE_NSLOT * KIE_SLOT_BYTES;

struct __align__(16) B1Shared {
    float rowacc[KIE_ROWACC_MAX];
    AttnSmem at;
    float red[64];
    int redi[32];
    uint64_t full[KIE_NSLOT];
    uint64_t empty[KIE_NSLOT];
    KieCmd cmd;
    volatile int abort;
    int token;
    int is_last;
    int gb_ok;
    int row0[KIE_NPH], row1[KIE_NPH];
};

struct Ring {
    uint8_t *base;
    uint32_t it;  // chunks consumed (consumers) or issued (producer) so far
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

// rows per ring chunk and 16-byte vectors per lane, both fixed by the row length K
__host__ __device__ inline int vec_per_lane(int K) {
    return K <= 2048 ? 1 : K <= 4096 ? 2 : K <= 8192 ? 4 : K <= 14336 ? 7 : 8;
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
            __threadfence();
            red_release_gpu_add_u64(P.bar, 1ull);
            uint64_t t0 = globaltimer();
            unsigned spins = 0;
            while (ld_acquire_gpu_u64(P.bar) < target) {
                if ((++spins & 255u) == 0) {
                    if (ld_volatile_u32(P.err) != 0u) { ok = 0; break; }
                    if ((long long)(globaltimer() - t0) > timeout_ns) {
                        set_error(P.err, DERR_BARRIER_TIMEOUT, where);
                        ok = 0;
                        break;
                    }
                }
            }
            __threadfence();
            if (!ok) S.abort = 1;
        }
        S.gb_ok = ok;
    }
    named_bar_sync(1, KIE_CONS_THREADS);
    return S.gb_ok != 0;
}

// --------------------------------------------------------------- producer

__device__ void produce(const KieParams &P, B1Shared &S, Ring &R, const KieCmd &cmd) {
    const int c = blockIdx.x;
    const uint8_t *seg = P.wpack + P.seg_off[c];
    long long phase_bytes[KIE_NPH];
    long long layer_bytes = 0;
    for (int ph = 0; ph < KIE_NPH; ph++) {
        phase_bytes[ph] = (long long)(S.row1[ph] - S.row0[ph]) * P.K[ph] * 2;
        if (ph != PH_HEAD) layer_bytes += phase_bytes[ph];
    }
    bool ok = true;
    for (int t = 0; t < cmd.n && ok; t++) {
        const bool head = (cmd.op != OP_PREFILL) || (t == cmd.n - 1);
        for (int l = 0; l <= P.L && ok; l++) {
            const bool is_head = (l == P.L);
            if (is_head && !head) break;
            const uint8_t *g = seg + (long long)l * layer_bytes;
            for (int ph = is_head ? PH_HEAD : 0; ph < (is_head ? KIE_NPH : PH_HEAD) && ok; ph++) {
                const int rows = S.row1[ph] - S.row0[ph];
                const int rb = P.K[ph] * 2, cr = P.cr[ph];
                for (int r = 0; r < rows; r += cr) {
                    const int nr = min(cr, rows - r);
                    const uint32_t bytes = (uint32_t)(nr * rb);
                    const uint32_t slot = R.it % KIE_NSLOT, par = (R.it / KIE_NSLOT) & 1u;
                    if (S.abort || !mbar_wait(&S.empty[slot], par ^ 1u, P.timeout_ns, &S.abort)) {
                        if (!S.abort) set_error(P.err, DERR_RING_TIMEOUT, 0x80);
                        S.abort = 1;
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&S.full[slot], bytes);
                    bulk_g2s(R.base + (size_t)slot * KIE_SLOT_BYTES, g, bytes, &S.full[slot]);
                    g += bytes;
                    R.it++;
                }
            }
        }
    }
    // Wait until every copy issued into the ring has landed before anyone may leave.
    const uint32_t first = R.it > KIE_NSLOT ? R.it - KIE_NSLOT : 0;
    for (uint32_t k = first; k < R.it; k++)
        mbar_wait(&S.full[k % KIE_NSLOT], (k / KIE_NSLOT) & 1u, P.timeout_ns, nullptr);
}

// --------------------------------------------------------------- consumer: GEMV phases

// input vector of a phase, element j
template <int DT>
__device__ __forceinline__ float phase_input(const KieParams &P, int ph, bool from_emb, int tok, int j) {
    if (ph == PH_O) return __ldcg(P.o + j);
    if (ph == PH_DOWN) return __ldcg(P.u + j);
    if (from_emb) return cvt1<DT>(P.emb[(size_t)tok * P.d + j]);
    return __ldcg(P.x + j);
}

// Runs one GEMV phase over this CTA's rows; row sums land in S.rowacc[0..rows).
template <int DT, int NV, int CR>
__device__ void gemv_phase(const KieParams &P, B1Shared &S, Ring &R, int ph, int l, int tok) {
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int K = P.K[ph];
    const int rows = S.row1[ph] - S.row0[ph];
    const bool norm = (ph == PH_QKV || ph == PH_GU || ph == PH_HEAD);
    const bool from_emb = (ph == PH_QKV && l == 0);

    float rstd = 1.f;
    if (norm) {
        float ss = 0.f;
        for (int j = tid; j < P.d; j += KIE_CONS_THREADS) {
            const float v = phase_input<DT>(P, ph, from_emb, tok, j);
            ss += v * v;
        }
        ss = warp_sum(ss);
        if (lane == 0) S.red[w] = ss;
        named_bar_sync(1, KIE_CONS_THREADS);
        if (w == 0) {
            float v = lane < KIE_CONS_WARPS ? S.red[lane] : 0.f;
            v = warp_sum(v);
            if (lane == 0) S.red[KIE_CONS_WARPS] = rsqrtf(v / (float)P.d + P.eps);
        }
        named_bar_sync(1, KIE_CONS_THREADS);
        rstd = S.red[KIE_CONS_WARPS];
    }
    const uint16_t *gain = P.gains + (size_t)(ph == PH_HEAD ? 2 * P.L : 2 * l + (ph == PH_GU ? 1 : 0)) * P.d;

    const int kslice = K >> 3;       // columns per warp
    const int nvec = K >> 6;         // 16-byte vectors per warp slice
    float h[NV][8];
#pragma unroll
    for (int i = 0; i < NV; i++) {
        const int v = lane + 32 * i;
#pragma unroll
        for (int e = 0; e < 8; e++) {
            float val = 0.f;
            if (v < nvec) {
                const int col = w * kslice + 8 * v + e;
                val = phase_input<DT>(P, ph, from_emb, tok, col);
                if (norm) val = val * rstd * cvt1<DT>(gain[col]);
            }
            h[i][e] = val;
        }
    }

    for (int r0 = 0; r0 < rows; r0 += CR) {
        const int nr = min(CR, rows - r0);
        const uint32_t slot = R.it % KIE_NSLOT, par = (R.it / KIE_NSLOT) & 1u;
        R.it++;
        bool have = !S.abort && mbar_wait(&S.full[slot], par, P.timeout_ns, &S.abort);
        have = __all_sync(0xffffffffu, have);  // one decision per warp (the reduction below needs all lanes)
        if (!have) {
            if (!S.abort) set_error(P.err, DERR_RING_TIMEOUT, (unsigned)ph);
            S.abort = 1;
            continue;  // keep the control flow; the command ends at the next barrier
        }
        const uint8_t *base = R.base + (size_t)slot * KIE_SLOT_BYTES + (size_t)w * kslice * 2;
        float acc[8];
#pragma unroll
        for (int r = 0; r < 8; r++) acc[r] = 0.f;
#pragma unroll
        for (int r = 0; r < CR; r++) {
            if (r < nr) {
                const uint8_t *rowp = base + (size_t)r * K * 2;
#pragma unroll
                for (int i = 0; i < NV; i++) {
                    const int v = lane + 32 * i;
                    if (v < nvec) {
                        const uint4 wv = *reinterpret_cast<const uint4 *>(rowp + v * 16);
                        float f[8];
                        cvt8<DT>(wv, f);
#pragma unroll
                        for (int e = 0; e < 8; e++) acc[r] = fmaf(f[e], h[i][e], acc[r]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[slot]);
        const float s = warp_reduce_rows<CR>(acc);
        constexpr int LPR = 32 / CR;
        if ((lane % LPR) == 0) {
            const int r = lane / LPR;
            if (r < nr) atomicAdd(&S.rowacc[r0 + r], s);
        }
    }
    named_bar_sync(1, KIE_CONS_THREADS);
}

template <int DT>
__device__ void gemv_dispatch(const KieParams &P, B1Shared &S, Ring &R, int ph, int l, int tok) {
    switch (vec_per_lane(P.K[ph])) {
        case 1: gemv_phase<DT, 1, 8>(P, S, R, ph, l, tok); break;
        case 2: gemv_phase<DT, 2, 4>(P, S, R, ph, l, tok); break;
        case 4: gemv_phase<DT, 4, 2>(P, S, R, ph, l, tok); break;
        case 7: gemv_phase<DT, 7, 1>(P, S, R, ph, l, tok); break;
        default: gemv_phase<DT, 8, 1>(P, S, R, ph, l, tok); break;
    }
}

// --------------------------------------------------------------- consumer: epilogues

// q/k rows come in rotation pairs (dim i, dim i + D/2); v rows use the same pairing.
template <int DT>
__device__ void epilogue_qkv(const KieParams &P, B1Shared &S, int l, int sid, int pos, int tok) {
    const int D = P.D, half = D >> 1, qd = P.Hq * D, kvd = P.Hkv * D;
    const int rbeg = S.row0[PH_QKV], npair = (S.row1[PH_QKV] - rbeg) >> 1;
    const float2 *rope = P.rope + (size_t)pos * half;
    const size_t sess = (size_t)sid * P.sess_stride;
    for (int p = threadIdx.x; p < npair; p += KIE_CONS_THREADS) {
        const int r = rbeg + 2 * p;
        float a = S.rowacc[2 * p], b = S.rowacc[2 * p + 1];
        S.rowacc[2 * p] = 0.f;
        S.rowacc[2 * p + 1] = 0.f;
        const int i = (r % D) >> 1;
        if (r < qd + kvd) {
            const float2 cs = rope[i];
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
    if (l == 0) {  // the residual starts as the embedding row (rows this CTA owns in the O phase)
        for (int r = S.row0[PH_O] + threadIdx.x; r < S.row1[PH_O]; r += KIE_CONS_THREADS)
            P.x[r] = cvt1<DT>(P.emb[(size_t)tok * P.d + r]);
    }
}

__device__ void epilogue_residual(const KieParams &P, B1Shared &S, int ph) {
    const int rbeg = S.row0[ph], n = S.row1[ph] - rbeg;
    for (int r = threadIdx.x; r < n; r += KIE_CONS_THREADS) {
        P.x[rbeg + r] = __ldcg(P.x + rbeg + r) + S.rowacc[r];
        S.rowacc[r] = 0.f;
    }
}

__device__ void epilogue_gu(const KieParams &P, B1Shared &S) {
    const int rbeg = S.row0[PH_GU], npair = (S.row1[PH_GU] - rbeg) >> 1;
    for (int p = threadIdx.x; p < npair; p += KIE_CONS_THREADS) {
        const float g = S.rowacc[2 * p], up = S.rowacc[2 * p + 1];
        S.rowacc[2 * p] = 0.f;
        S.rowacc[2 * p + 1] = 0.f;
        P.u[(rbeg >> 1) + p] = g / (1.f + expf(-g)) * up;
    }
}

__device__ __forceinline__ void argmax_combine(float &v, int &i, float v2, int i2) {
    if (v2 > v || (v2 == v && i2 < i)) { v = v2; i = i2; }
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
__device__ void epilogue_head(const KieParams &P, B1Shared &S, float *logits) {
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int rbeg = S.row0[PH_HEAD], n = S.row1[PH_HEAD] - rbeg;
    float bv = -CUDART_INF_F;
    int bi = 0x7fffffff;
    for (int r = tid; r < n; r += KIE_CONS_THREADS) {
        const float v = S.rowacc[r];
        S.rowacc[r] = 0.f;
        if (logits) logits[rbeg + r] = v;
        argmax_combine(bv, bi, v, rbeg + r);
    }
    warp_argmax(bv, bi);
    if (lane == 0) { S.red[w] = bv; S.redi[w] = bi; }
    named_bar_sync(1, KIE_CONS_THREADS);
    if (w == 0) {
        float v = lane < KIE_CONS_WARPS ? S.red[lane] : -CUDART_INF_F;
        int i = lane < KIE_CONS_WARPS ? S.redi[lane] : 0x7fffffff;
        warp_argmax(v, i);
        if (lane == 0) { P.cand_val[blockIdx.x] = v; P.cand_idx[blockIdx.x] = i; }
    }
}

// after the head barrier: every CTA reduces all candidates to the same token
__device__ int final_argmax(const KieParams &P, B1Shared &S) {
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    float v = -CUDART_INF_F;
    int i = 0x7fffffff;
    for (int c = tid; c < P.nblk; c += KIE_CONS_THREADS) argmax_combine(v, i, __ldcg(P.cand_val + c), __ldcg(P.cand_idx + c));
    warp_argmax(v, i);
    if (lane == 0) { S.red[w] = v; S.redi[w] = i; }
    named_bar_sync(1, KIE_CONS_THREADS);
    if (w == 0) {
        v = lane < KIE_CONS_WARPS ? S.red[lane] : -CUDART_INF_F;
        i = lane < KIE_CONS_WARPS ? S.redi[lane] : 0x7fffffff;
        warp_argmax(v, i);
        if (lane == 0) S.token = i;
    }
    named_bar_sync(1, KIE_CONS_THREADS);
    return S.token;
}

// --------------------------------------------------------------- consumer: attention

template <int DT>
__device__ void attention_layer(const KieParams &P, B1Shared &S, int l, int sid, int pos) {
    AttnArgs A;
    A.q = P.q;
    A.k = P.kcache + (size_t)sid * P.sess_stride + (size_t)l * P.Hkv * P.max_ctx * P.D;
    A.v = P.vcache + (size_t)sid * P.sess_stride + (size_t)l * P.Hkv * P.max_ctx * P.D;
    A.head_stride = (long long)P.max_ctx * P.D;
    A.part = P.part;
    A.cnt = P.cnt;
    A.o = P.o;
    A.D = P.D;
    A.Hkv = P.Hkv;
    A.nsplit = P.splits;
    A.ctx = pos + 1;
    attn_all_units<DT>(A, S.at, P.G, blockIdx.x, P.nblk);
}

// --------------------------------------------------------------- consumer: one command

template <int DT>
__device__ void consume(const KieParams &P, B1Shared &S, Ring &R, const KieCmd &cmd, unsigned long long &epoch) {
    int tok = cmd.in_tok;
    if (cmd.op == OP_DECODE && cmd.tok_dev) tok = __ldcg(cmd.tok_dev);
    for (int t = 0; t < cmd.n; t++) {
        const int pos = cmd.pos0 + t;
        if (cmd.op == OP_PREFILL) tok = __ldcg(P.tokbuf + t);
        if (tok < 0 || tok >= P.V) {
            if (threadIdx.x == 0) set_error(P.err, DERR_BAD_TOKEN, 0);
            S.abort = 1;
        }
        const bool head = (cmd.op != OP_PREFILL) || (t == cmd.n - 1);
        for (int l = 0; l < P.L; l++) {
            gemv_dispatch<DT>(P, S, R, PH_QKV, l, tok);
            epilogue_qkv<DT>(P, S, l, cmd.sid, pos, tok);
            grid_barrier(P, S, epoch, P.timeout_ns, 1);
            if (!S.abort) attention_layer<DT>(P, S, l, cmd.sid, pos);
            grid_barrier(P, S, epoch, P.timeout_ns, 2);
            gemv_dispatch<DT>(P, S, R, PH_O, l, tok);
            epilogue_residual(P, S, PH_O);
            grid_barrier(P, S, epoch, P.timeout_ns, 3);
            gemv_dispatch<DT>(P, S, R, PH_GU, l, tok);
            epilogue_gu(P, S);
            grid_barrier(P, S, epoch, P.timeout_ns, 4);
            gemv_dispatch<DT>(P, S, R, PH_DOWN, l, tok);
            epilogue_residual(P, S, PH_DOWN);
            grid_barrier(P, S, epoch, P.timeout_ns, 5);
        }
        if (head) {
            gemv_dispatch<DT>(P, S, R, PH_HEAD, P.L, tok);
            float *lg = nullptr;
            if (cmd.logits) lg = cmd.logits + (cmd.op == OP_PREFILL ? 0 : (size_t)t * P.V);
            epilogue_head(P, S, lg);
            grid_barrier(P, S, epoch, P.timeout_ns, 6);
            tok = final_argmax(P, S);
            if (blockIdx.x == 0 && threadIdx.x == 0 && cmd.out) cmd.out[cmd.op == OP_PREFILL ? 0 : t] = tok;
        }
    }
}

// --------------------------------------------------------------- the kernel

template <int DT>
__global__ void __launch_bounds__(KIE_THREADS, 1) kie_b1_kernel(KieParams P, KieCmd one, int resident) {
    extern __shared__ __align__(1024) uint8_t smem[];
    B1Shared &S = *reinterpret_cast<B1Shared *>(smem + RING_BYTES);
    const int tid = threadIdx.x;
    if (tid == 0) {
        for (int i = 0; i < KIE_NSLOT; i++) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], KIE_CONS_WARPS);
        }
        fence_mbar_init();
        S.abort = 0;
    }
    for (int i = tid; i < KIE_ROWACC_MAX; i += KIE_THREADS) S.rowacc[i] = 0.f;
    attn_smem_init(S.at, tid, KIE_THREADS);
    if (tid < KIE_NPH) {
        S.row0[tid] = P.row0[tid * (P.nblk + 1) + blockIdx.x];
        S.row1[tid] = P.row0[tid * (P.nblk + 1) + blockIdx.x + 1];
    }
    __syncthreads();

    Ring R{smem, 0};
    unsigned long long epoch = 0;
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
            if (tid == KIE_CONS_THREADS) produce(P, S, R, cmd);
        } else {
            consume<DT>(P, S, R, cmd, epoch);
        }
        __syncthreads();
        if (resident && blockIdx.x == 0 && tid == 0) {
            __threadfence_system();
            P.mbox->status = S.abort ? -1 : 0;
            st_release_sys_u32(&P.mbox->done_seq, cmd.seq);
        }
        if (!resident || S.abort) break;
    }
}

}  // namespace

// --------------------------------------------------------------- host-side launch helpers

extern "C++" {

size_t kie_b1_smem_bytes() { return RING_BYTES + sizeof(B1Shared); }

int kie_b1_vec_per_lane(int K) { return vec_per_lane(K); }

cudaError_t kie_b1_prepare(int dtype) {
    const size_t smem = kie_b1_smem_bytes();
    cudaError_t e = dtype == KIE_BF16
                        ? cudaFuncSetAttribute(kie_b1_kernel<KIE_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                        : cudaFuncSetAttribute(kie_b1_kernel<KIE_FP16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return e;
}

cudaError_t kie_b1_occupancy(int dtype, int *blocks_per_sm) {
    const size_t smem = kie_b1_smem_bytes();
    return dtype == KIE_BF16
               ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, kie_b1_kernel<KIE_BF16>, KIE_THREADS, smem)
               : cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, kie_b1_kernel<KIE_FP16>, KIE_THREADS, smem);
}

cudaError_t kie_b1_launch(const KieParams &P, const KieCmd &one, int resident, cudaStream_t stream) {
    KieParams p = P;
    KieCmd c = one;
    int r = resident;
    void *args[] = {&p, &c, &r};
    const void *fn = P.dtype == KIE_BF16 ? (const void *)kie_b1_kernel<KIE_BF16> : (const void *)kie_b1_kernel<KIE_FP16>;
    return cudaLaunchCooperativeKernel(fn, dim3(P.nblk), dim3(KIE_THREADS), args, kie_b1_smem_bytes(), stream);
}

}  // extern "C++"
