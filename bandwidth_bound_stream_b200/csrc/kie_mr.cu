// Multi-row decode megakernel for sm_100a: the continuous-inference tick and chunked prefill.
//
// All sessions due on a tick advance as one batch, so every weight byte is read once for
// the whole group ("实时AI推理为何贵56倍？持续推理与常驻内核的破局之道", section 让所有活跃会话同步推进),
// by one resident program (section 让工作常驻 GPU) with a schedule fixed ahead of time (section
// 把一切提前决定好). With up to 64 rows (sessions, or consecutive positions of one session in
// prefill) per step, each weight contraction Y[rows][N] = X[rows][K] W[N][K]^T runs on the
// 5th-generation tensor cores:
//
//   D[128 weight rows][128] (fp32, TMEM) += A[128 weight rows][64] * B[128][64]^T  per k-step
//
// A is a 128 x 64 weight tile, stored in HBM already in the K-major 128-byte-swizzled layout
// the MMA reads, and streamed by the producer warp with 1-D bulk copies, two tiles (32 KB) per
// copy, into a ring of four such atoms.
// B holds the activations split into two 16-bit halves: rows 0-63 carry hi(x) and rows
// 64-127 carry lo(x) = x - hi(x), so D[:, s] + D[:, 64 + s] equals W x_s to about 16 bits of
// the fp32 activation (the tensor cores take 16-bit operands only). The phase that finalises
// an activation writes it once, already in that tile layout, to a small global buffer (one
// tile per k-step: the RMSNorm phases for QKV, gate/up and the head, attention for O, the
// activation phase silu(gate)*up for down); during the GEMM, thread 0 streams the tile of
// each k-step from there (L2) into a ring of two atoms with bulk copies, beside the weight tiles.
// Warp 8 issues tcgen05.mma and commits, warps 4-7 read the accumulator from TMEM and add
// it into the fp32 outputs with atomics: the weight tiles of one phase are split evenly over
// the SMs by k-steps, so partial sums of a row block from several SMs meet in global memory.
//
// Phases per layer, each ended by a grid barrier: NORM1 (per-row 1/rms -> QKV operand, clear
// the QKV accumulator) | QKV | ROPE (rotate q and k, append K and V) | ATTN (-> O operand) |
// O (+= residual) | NORM2 | GATE/UP | ACT | DOWN (+= residual); then NORMF | HEAD | ARGMAX
// per step. Attention puts both of its products on the tensor cores as well (see the
// tensor-core attention below), with warp 8 issuing them between the QKV and O projections.
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kie_attn.cuh"
#include "kie_device.cuh"
#include "kie_sample.cuh"

namespace {

constexpr int MR_THREADS = 320;           // warps 0-3 (thread 0: B loads), 4-7 epilogue, 8 MMA, 9 producer
constexpr int MR_WORKERS = 256;           // warps 0-7 also run the non-GEMM phases
constexpr int TILE = 16384;               // one 128 x 64 16-bit tile
// A GEMM "atom" is the tiles of two consecutive 64-wide k-steps of one 128-row block (one when
// it is the odd last k-step of the block), moved with one 32 KB bulk copy: on B200 a ring of
// 4 x 32 KB copies streams ~7.3 TB/s where 8 x 16 KB copies stream ~5.8 TB/s.
constexpr int ATOM = 2 * TILE;
constexpr int A_SLOTS = 4, B_SLOTS = 2;   // atoms in flight: weights (HBM), activations (L2)
constexpr int KV_SLOTS = 4;               // 16 KB K/V chunks of the CUDA-core attention, in the B ring
constexpr int MAXR = 64;                  // rows per step (hi half of B; lo half at +64)
constexpr int TMEM_COLS = 256;            // two 128-column fp32 accumulators
constexpr int NU_MAX = 16;                // units per attention stream (a CTA with more runs several)
constexpr int AT_STAGES = 3;              // K/V tile stages of the tensor-core attention (A ring x 2, B ring)
constexpr int AS_MAX = 2048;              // (unit, pass) entries the longest-first assignment sorts
constexpr int AS_LIST = 16;               // ... entries per CTA it can hand out (>= AS_MAX / 148, rounded up)

enum { G_QKV = 0, G_O = 1, G_GU = 2, G_DOWN = 3, G_HEAD = 4, NG = 5 };

struct __align__(1024) MrShared {
    uint8_t a[A_SLOTS][ATOM];
    uint8_t b[B_SLOTS][ATOM];
    AttnSmem at;
    uint64_t a_full[A_SLOTS], a_empty[A_SLOTS], b_full[B_SLOTS], b_empty[B_SLOTS];
    uint64_t acc_full[2], acc_empty[2], drain;
    uint64_t k_full[KV_SLOTS], k_empty[KV_SLOTS];  // the B ring as a K/V chunk ring in attention
    uint32_t k_iss;                              // K/V chunks issued so far (thread 0)
    // tensor-core attention: K, V tile per stage; scores done; scores read (softmax threads);
    // per P.V buffer: Pt and correction in (softmax threads), product done, product read
    // (output threads); a unit's query operand in; a stream's table in
    uint64_t at_k[AT_STAGES], at_v[AT_STAGES], at_s, at_sf, at_p[2], at_o[2], at_of[2], at_q, at_tab;
    uint32_t tk_iss[AT_STAGES], tv_iss[AT_STAGES];  // tile copies issued
    float at_corr[2][KIE_GMAX];                  // per tile (two in flight): rescale of the running sums
    float at_l[4][KIE_GMAX];                     // the softmax warps' shares of the sums
    long long un_row0[NU_MAX];                   // the attention stream's units: first K/V arena row,
    int un_ctx[NU_MAX], un_nt[NU_MAX];           // context, tiles
    int un_n, un_more;                           // units in the stream; another stream follows
    int un_cnt;                                  // this CTA's (unit, pass) entries this step (-1: dealt in turn)
    uint16_t un_list[AS_LIST];                   // ... and which, longest first
    volatile uint32_t att_seq;                   // attention phases finished (the producer waits on it)
    uint32_t tmem_base;
    KieCmd cmd;
    volatile int abort;
    int gb_ok;
    int a0[NG], a1[NG];
    float red[32];
};

// ------------------------------------------------------------------ tcgen05 / TMEM helpers

KIE_DEV void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
KIE_DEV void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
KIE_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
KIE_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
KIE_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
KIE_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 2-D tiled bulk tensor copy (TMA, no multicast) of box (x, y) of the tensor map into shared
// memory, completion as transaction bytes on `bar`
KIE_DEV void tma_load_2d(void *dst, const void *tmap, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// D[tmem] (+)= A(desc) * B(desc)^T, M = 128, N from the instruction descriptor, K = 16 (16-bit inputs, fp32 accumulate)
KIE_DEV void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// arrive on `bar` once every tcgen05 operation issued so far by this thread has completed
KIE_DEV void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 consecutive fp32 columns from TMEM
KIE_DEV void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
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
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 16 consecutive fp32 columns from TMEM
KIE_DEV void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; i++) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor of a K-major, 128-byte-swizzled tile (8-row atoms of 1024 B).
KIE_DEV uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);       // start address
    d |= (uint64_t)1u << 16;                        // leading byte offset (unused when swizzled)
    d |= (uint64_t)(1024u >> 4) << 32;              // stride byte offset: next 8-row atom
    d |= (uint64_t)1u << 46;                        // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                        // layout: 128-byte swizzle
    return d;
}

// Shared-memory matrix descriptor of an MN-major, 128-byte-swizzled operand as a 2-D tile
// copy of 64-element-wide boxes lands it: 128-byte rows of 64 consecutive M elements, one row
// per k, 8-row atoms of 1024 B; the next 64 M elements lie one box (TILE bytes) further on.
KIE_DEV uint64_t smem_desc_mn_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);       // start address
    d |= (uint64_t)((TILE >> 4) & 0x3FFFu) << 16;   // leading byte offset: next 64 elements of M
    d |= (uint64_t)(1024u >> 4) << 32;              // stride byte offset: next 8 rows of K
    d |= (uint64_t)1u << 46;                        // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                        // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor: fp32 accumulate, A and B 16-bit (f16 or bf16), both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_f16(int dtype, uint32_t n = 128) {
    return (1u << 4) | ((uint32_t)(dtype == KIE_BF16) << 7) | ((uint32_t)(dtype == KIE_BF16) << 10) |
           ((n >> 3) << 17) | ((128u >> 4) << 24);
}

// ------------------------------------------------------------------ shared helpers

struct Gemm {
    int N, K, ldy;
    float *y;
};

__device__ __forceinline__ Gemm gemm_of(const KieParams &P, int g) {
    Gemm G;
    switch (g) {
        case G_QKV: G = {P.Hq * P.D + 2 * P.Hkv * P.D, P.d, P.Hq * P.D + 2 * P.Hkv * P.D, P.mr_yqkv}; break;
        case G_O: G = {P.d, P.Hq * P.D, P.d, P.mr_x}; break;
        case G_GU: G = {2 * P.F, P.d, 2 * P.F, P.mr_ygu}; break;
        case G_DOWN: G = {P.d, P.F, P.d, P.mr_x}; break;
        default: G = {P.V, P.d, P.V, P.mr_logits}; break;
    }
    return G;
}

// atoms per row block of a K-long contraction, and the tiles (1 or 2) of atom a
__device__ __forceinline__ int atoms_per_rb(int K) { return (K / 64 + 1) / 2; }
__device__ __forceinline__ int atom_tiles(int K, int a) { return min(2, K / 64 - 2 * (a % atoms_per_rb(K))); }

// words of a command record (volatile: it may live in mapped host memory)
__device__ __forceinline__ void copy_cmd(KieCmd *dst, const KieCmd *src, bool vol) {
    uint32_t *d = reinterpret_cast<uint32_t *>(dst);
    if (vol) {
        const volatile uint32_t *s = reinterpret_cast<const volatile uint32_t *>(src);
        for (int i = 0; i < (int)(sizeof(KieCmd) / 4); i++) d[i] = s[i];
    } else {
        const uint32_t *s = reinterpret_cast<const uint32_t *>(src);
        for (int i = 0; i < (int)(sizeof(KieCmd) / 4); i++) d[i] = __ldcg(s + i);
    }
}

// grid barrier over warps 0-7 of every CTA (bounded; see the batch-1 kernel)
__device__ bool mr_barrier(const KieParams &P, MrShared &S, unsigned long long &epoch, long long timeout_ns,
                           unsigned where) {
    fence_proxy_async_global();  // B-operand tiles written before the barrier are read by bulk copies after it
    named_bar_sync(1, MR_WORKERS);
    if (threadIdx.x == 0) {
        int ok = !S.abort;
        if (ok) {
            epoch += 1;
            const unsigned long long target = epoch * (unsigned long long)P.nblk;
            red_release_gpu_add_u64(P.bar, 1ull);
            const uint64_t t0 = globaltimer();
            unsigned spins = 0;
            while (ld_acquire_gpu_u64(P.bar) < target) {
                if ((++spins & 255u) == 0) {
                    if (ld_volatile_u32(P.err) != 0u) {
                        ok = 0;
                        break;
                    }
                    if ((long long)(globaltimer() - t0) > timeout_ns) {
                        set_error(P.err, DERR_BARRIER_TIMEOUT, 0x40 | where);
                        ok = 0;
                        break;
                    }
                }
            }
            if (!ok) S.abort = 1;
        }
        S.gb_ok = ok;
    }
    named_bar_sync(1, MR_WORKERS);
    return S.gb_ok != 0;
}

__device__ __forceinline__ bool head_needed(const KieCmd &cmd) { return cmd.op == OP_TICK || (cmd.flags & 1); }

// the GEMM phases of one step, in stream order
__device__ __forceinline__ int steps_of(const KieCmd &cmd) { return cmd.op == OP_TICK ? cmd.n : 1; }

// ------------------------------------------------------------------ producer (warp 9)

__device__ void mr_produce(const KieParams &P, MrShared &S, uint32_t &a_it, uint32_t &o_seq, const KieCmd &cmd) {
    const uint8_t *seg = P.mr_wpack + P.mr_seg_off[blockIdx.x];
    const int steps = steps_of(cmd);
    for (int st = 0; st < steps && !S.abort; st++) {
        const uint8_t *src = seg;
        for (int l = 0; l <= P.L && !S.abort; l++) {
            if (l == P.L && !head_needed(cmd)) break;
            for (int g = (l < P.L ? 0 : G_HEAD); g < (l < P.L ? G_HEAD : NG); g++) {
                const int K = gemm_of(P, g).K;
                if (g == G_O) {  // attention uses the ring as its K/V buffers: wait until it is done
                    const uint64_t t0 = globaltimer();
                    while (S.att_seq <= o_seq && !S.abort) {
                        if ((long long)(globaltimer() - t0) > P.timeout_ns) {
                            set_error(P.err, DERR_RING_TIMEOUT, 0x98);
                            S.abort = 1;
                        }
                        __nanosleep(64);
                    }
                    o_seq++;
                    fence_proxy_async_smem();  // attention's generic reads of the ring, then these copies
                }
                for (int a = S.a0[g]; a < S.a1[g]; a++) {
                    const uint32_t slot = a_it % A_SLOTS, par = (a_it / A_SLOTS) & 1u;
                    const uint32_t bytes = (uint32_t)atom_tiles(K, a) * TILE;
                    if (S.abort || !mbar_wait(&S.a_empty[slot], par ^ 1u, P.timeout_ns, &S.abort)) {
                        if (!S.abort) set_error(P.err, DERR_RING_TIMEOUT, 0x90);
                        S.abort = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&S.a_full[slot], bytes);
                    bulk_g2s(S.a[slot], src, bytes, &S.a_full[slot]);
                    src += bytes;
                    a_it++;
                }
            }
        }
    }
    // every issued copy must land before the CTA may leave
    const uint32_t first = a_it > A_SLOTS ? a_it - A_SLOTS : 0;
    for (uint32_t k = first; k < a_it; k++) mbar_wait(&S.a_full[k % A_SLOTS], (k / A_SLOTS) & 1u, P.timeout_ns, nullptr);
}

// ------------------------------------------------------------------ MMA issuer (warp 8, one lane)

__device__ bool mr_attn_mma(const KieParams &P, MrShared &S, int M, unsigned long long &at_it, uint32_t &q_it,
                            uint32_t &tab_it);

__device__ void mr_mma(const KieParams &P, MrShared &S, uint32_t &a_it, uint32_t &b_it, uint32_t &u_it,
                       unsigned long long &at_it, uint32_t &q_it, uint32_t &tab_it, const KieCmd &cmd) {
    const uint32_t idesc = idesc_f16(P.dtype);
    const int steps = steps_of(cmd);
    bool ok = true;
    for (int st = 0; st < steps && ok; st++) {
        for (int l = 0; l <= P.L && ok; l++) {
            if (l == P.L && !head_needed(cmd)) break;
            for (int g = (l < P.L ? 0 : G_HEAD); g < (l < P.L ? G_HEAD : NG) && ok; g++) {
                // the tensor-core attention runs between the QKV and O projections
                if (g == G_O && P.mr_kmap && !mr_attn_mma(P, S, cmd.n_sess, at_it, q_it, tab_it)) {
                    ok = false;
                    break;
                }
                const int K = gemm_of(P, g).K, natk = atoms_per_rb(K);
                int cur_rb = -1;
                uint32_t ab = 0;
                for (int a = S.a0[g]; a < S.a1[g] && ok; a++) {
                    const int rb = a / natk, nt = atom_tiles(K, a);
                    const bool first = (rb != cur_rb);
                    if (first) {  // new unit: take a free accumulator
                        cur_rb = rb;
                        ab = u_it & 1u;
                        if (!mbar_wait(&S.acc_empty[ab], ((u_it >> 1) & 1u) ^ 1u, P.timeout_ns, &S.abort)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    const uint32_t as = a_it % A_SLOTS, bs = b_it % B_SLOTS;
                    if (!mbar_wait(&S.a_full[as], (a_it / A_SLOTS) & 1u, P.timeout_ns, &S.abort) ||
                        !mbar_wait(&S.b_full[bs], (b_it / B_SLOTS) & 1u, P.timeout_ns, &S.abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(S.a[as]), sb = smem_u32(S.b[bs]);
                    const uint32_t tmem_d = S.tmem_base + ab * 128u;
                    for (int t = 0; t < nt; t++)
#pragma unroll
                        for (int kk = 0; kk < 4; kk++)
                            umma_f16(tmem_d, smem_desc_sw128(sa + t * TILE + kk * 32), smem_desc_sw128(sb + t * TILE + kk * 32),
                                     idesc, (first && t == 0 && kk == 0) ? 0u : 1u);
                    umma_commit(&S.a_empty[as]);
                    umma_commit(&S.b_empty[bs]);
                    a_it++;
                    b_it++;
                    const bool last = (a + 1 == S.a1[g]) || ((a + 1) / natk != rb);
                    if (last) {
                        umma_commit(&S.acc_full[ab]);
                        u_it++;
                    }
                }
            }
        }
    }
    if (!ok) {
        if (!S.abort) set_error(P.err, DERR_MMA_TIMEOUT, 0x91);
        S.abort = 1;
    }
    // all MMAs issued by this thread must finish before TMEM or the rings are released
    umma_commit(&S.drain);
}

// ------------------------------------------------------------------ B operand

// hi/lo 16-bit halves of 8 consecutive activations -> chunk c of row m (hi) and 64 + m (lo)
// of a swizzled B tile
template <int DT>
__device__ __forceinline__ void put_b8(uint8_t *tile, int m, int c, const float (&v)[8]) {
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const float x0 = v[2 * j], x1 = v[2 * j + 1];
        const uint16_t h0 = store1<DT>(x0), h1 = store1<DT>(x1);
        const uint16_t l0 = store1<DT>(x0 - cvt1<DT>(h0)), l1 = store1<DT>(x1 - cvt1<DT>(h1));
        hw[j] = (uint32_t)h0 | ((uint32_t)h1 << 16);
        lw[j] = (uint32_t)l0 | ((uint32_t)l1 << 16);
    }
    *reinterpret_cast<uint4 *>(tile + sw128(m, c)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4 *>(tile + sw128(MAXR + m, c)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
}

// Thread 0 during a GEMM phase: the B tile of every k-step this CTA multiplies, in atom
// order, from the global operand buffer into the B ring (finished by the phase before, and
// made visible by the grid barrier in between).
__device__ void mr_bload(const KieParams &P, MrShared &S, uint32_t &b_it, int g) {
    const int K = gemm_of(P, g).K, natk = atoms_per_rb(K);
    fence_proxy_async_global();
    fence_proxy_async_smem();  // attention read the B ring through the generic proxy
    for (int a = S.a0[g]; a < S.a1[g]; a++) {
        const uint32_t bs = b_it % B_SLOTS;
        if (S.abort || !mbar_wait(&S.b_empty[bs], ((b_it / B_SLOTS) & 1u) ^ 1u, P.timeout_ns, &S.abort)) {
            if (!S.abort) set_error(P.err, DERR_RING_TIMEOUT, 0x92);
            S.abort = 1;
            return;
        }
        const uint32_t bytes = (uint32_t)atom_tiles(K, a) * TILE;
        mbar_arrive_expect_tx(&S.b_full[bs], bytes);
        bulk_g2s(S.b[bs], P.mr_bpack + (size_t)(2 * (a % natk)) * TILE, bytes, &S.b_full[bs]);
        b_it++;
    }
}

// ------------------------------------------------------------------ epilogue (warps 4-7)

__device__ void mr_epilogue(const KieParams &P, MrShared &S, uint32_t &u_it, int g, int M) {
    const Gemm G = gemm_of(P, g);
    const int natk = atoms_per_rb(G.K);
    const int wq = (threadIdx.x >> 5) & 3, lane = threadIdx.x & 31;
    int cur_rb = -1;
    for (int a = S.a0[g]; a < S.a1[g]; a++) {
        const int rb = a / natk;
        if (rb == cur_rb) continue;
        cur_rb = rb;
        const uint32_t ab = u_it & 1u;
        bool ok = !S.abort && mbar_wait(&S.acc_full[ab], (u_it >> 1) & 1u, P.timeout_ns, &S.abort);
        ok = __all_sync(0xffffffffu, ok);
        u_it++;
        if (!ok) {
            if (!S.abort) set_error(P.err, DERR_MMA_TIMEOUT, 0x93);
            S.abort = 1;
            continue;
        }
        tc_fence_after();
        const int row = rb * 128 + wq * 32 + lane;
        const uint32_t taddr = S.tmem_base + ab * 128u + ((uint32_t)(wq * 32) << 16);
#pragma unroll 1
        for (int half = 0; half < 2; half++) {
            float hi[32], lo[32];
            tmem_ld32(taddr + half * 32, hi);
            tmem_ld32(taddr + 64 + half * 32, lo);
            if (row < G.N) {
#pragma unroll
                for (int j = 0; j < 32; j++) {
                    const int s = half * 32 + j;
                    if (s < M && in_bounds(s < MAXR && row < G.ldy, P.err, 0x23))
                        atomicAdd(G.y + (size_t)s * G.ldy + row, hi[j] + lo[j]);
                }
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.acc_empty[ab]);
    }
}

// ------------------------------------------------------------------ worker phases (warps 0-7)

// Per row (one CTA per row): 1/rms of the residual, then the row of the next GEMM's B operand,
// x * (1/rms) * gain, in 8-column chunks (the second pass re-reads the row from L2, which
// keeps the register budget of the 10-warp CTA); also clears the next GEMM's accumulator.
template <int DT>
__device__ void phase_norm(const KieParams &P, MrShared &S, int g_next, int l, bool load_emb, int M) {
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    if (g_next != G_O) {  // clear rows 0..M-1 of the accumulator of the next GEMM
        const Gemm G = gemm_of(P, g_next);
        const size_t n = (size_t)M * G.ldy;
        for (size_t i = (size_t)blockIdx.x * MR_WORKERS + tid; i < n; i += (size_t)P.nblk * MR_WORKERS) G.y[i] = 0.f;
    }
    const int nch = P.d >> 3;
    const uint16_t *gain = P.gains + (size_t)(g_next == G_HEAD ? 2 * P.L : 2 * l + (g_next == G_GU ? 1 : 0)) * P.d;
    for (int m = blockIdx.x; m < M; m += P.nblk) {
        float *x = P.mr_x + (size_t)m * P.d;
        float ss = 0.f;
        if (load_emb) {  // a new step starts from the embedding rows of its input tokens
            int tok = __ldcg(P.mr_tok + m);
            if (tok < 0 || tok >= P.V) {  // e.g. an argmax over non-finite logits: fail the command
                if (tid == 0) set_error(P.err, DERR_BAD_TOKEN, 0x40);
                S.abort = 1;
                tok = 0;
            }
            for (int c = tid; c < nch; c += MR_WORKERS) {
                float v[8];
                cvt8<DT>(__ldg(reinterpret_cast<const uint4 *>(P.emb + (size_t)tok * P.d + 8 * c)), v);
                float4 *xd = reinterpret_cast<float4 *>(x + 8 * c);
                xd[0] = make_float4(v[0], v[1], v[2], v[3]);
                xd[1] = make_float4(v[4], v[5], v[6], v[7]);
#pragma unroll
                for (int e = 0; e < 8; e++) ss += v[e] * v[e];
            }
        } else {
            for (int c = tid; c < nch; c += MR_WORKERS) {
                const float4 a = __ldcg(reinterpret_cast<const float4 *>(x + 8 * c));
                const float4 b = __ldcg(reinterpret_cast<const float4 *>(x + 8 * c + 4));
                ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w + b.x * b.x + b.y * b.y + b.z * b.z + b.w * b.w;
            }
        }
        ss = warp_sum(ss);
        if (lane == 0) S.red[w] = ss;
        named_bar_sync(1, MR_WORKERS);
        float tot = 0.f;
        for (int k = 0; k < MR_WORKERS / 32; k++) tot += S.red[k];
        const float r = rsqrtf(tot / (float)P.d + P.eps);
        named_bar_sync(1, MR_WORKERS);
        for (int c = tid; c < nch; c += MR_WORKERS) {
            const float4 a = __ldcg(reinterpret_cast<const float4 *>(x + 8 * c));
            const float4 b = __ldcg(reinterpret_cast<const float4 *>(x + 8 * c + 4));
            float gv[8];
            cvt8<DT>(__ldg(reinterpret_cast<const uint4 *>(gain + 8 * c)), gv);
            const float v[8] = {a.x * r * gv[0], a.y * r * gv[1], a.z * r * gv[2], a.w * r * gv[3],
                                b.x * r * gv[4], b.y * r * gv[5], b.z * r * gv[6], b.w * r * gv[7]};
            if (in_bounds(m < MAXR && (c >> 3) < max(max(P.d, P.Hq * P.D), P.F) / 64, P.err, 0x24))
                put_b8<DT>(P.mr_bpack + (size_t)(c >> 3) * TILE, m, c & 7, v);
        }
    }
}

// the down projection's operand: u = silu(gate) * up, all rows, spread over every CTA
template <int DT>
__device__ void phase_act(const KieParams &P, int M) {
    const int nch = P.F >> 3;
    const long long n = (long long)M * nch;
    for (long long i = (long long)blockIdx.x * MR_WORKERS + threadIdx.x; i < n; i += (long long)P.nblk * MR_WORKERS) {
        const int m = (int)(i / nch), c = (int)(i % nch);
        const float *gs = P.mr_ygu + (size_t)m * 2 * P.F + 8 * c;
        const float *us = gs + P.F;
        float v[8];
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const float4 a = __ldcg(reinterpret_cast<const float4 *>(gs + 4 * h));
            const float4 b = __ldcg(reinterpret_cast<const float4 *>(us + 4 * h));
            const float ga[4] = {a.x, a.y, a.z, a.w}, ub[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int e = 0; e < 4; e++) v[4 * h + e] = ga[e] / (1.f + expf(-ga[e])) * ub[e];
        }
        if (in_bounds(m < MAXR && (c >> 3) < max(max(P.d, P.Hq * P.D), P.F) / 64, P.err, 0x25))
            put_b8<DT>(P.mr_bpack + (size_t)(c >> 3) * TILE, m, c & 7, v);
    }
}

// rotate q and k of every row, store q, append k and v to each row's cache at its position
template <int DT>
__device__ void phase_rope(const KieParams &P, int l, int M) {
    const int D = P.D, half = D >> 1, qd = P.Hq * D, kvd = P.Hkv * D, ldy = qd + 2 * kvd;
    const int pairs = (P.Hq + P.Hkv) * half + P.Hkv * half;  // q pairs, k pairs, v pairs
    for (int m = blockIdx.x; m < M; m += P.nblk) {
        const int sid = __ldcg(P.mr_sid + m), pos = __ldcg(P.mr_pos + m);
        const float *y = P.mr_yqkv + (size_t)m * ldy;
        const size_t sess = (size_t)sid * P.sess_stride;
        for (int p = threadIdx.x; p < pairs; p += MR_WORKERS) {
            const int head = p / half, i = p % half;  // heads: q 0..Hq-1, k Hq.., v Hq+Hkv..
            const int base = head * D;                 // column of the head in y (q | k | v)
            const float a = __ldcg(y + base + i), b = __ldcg(y + base + i + half);
            if (head < P.Hq + P.Hkv) {
                const float2 cs = P.rope[(size_t)pos * half + i];
                const float ra = a * cs.x - b * cs.y, rb = b * cs.x + a * cs.y;
                if (head < P.Hq) {
                    float *q = P.mr_q + (size_t)m * qd + base;
                    if (in_bounds(m < MAXR && base + i + half < qd, P.err, 0x20)) {
                        q[i] = ra;
                        q[i + half] = rb;
                    }
                } else {
                    const int g = head - P.Hq;
                    uint16_t *kp = P.kcache + sess + ((size_t)(l * P.Hkv + g) * P.max_ctx + pos) * D;
                    if (in_bounds(pos < P.max_ctx && g < P.Hkv && i + half < D, P.err, 0x21)) {
                        kp[i] = store1<DT>(ra);
                        kp[i + half] = store1<DT>(rb);
                    }
                }
            } else {
                const int g = head - P.Hq - P.Hkv;
                uint16_t *vp = P.vcache + sess + ((size_t)(l * P.Hkv + g) * P.max_ctx + pos) * D;
                if (in_bounds(pos < P.max_ctx && g < P.Hkv && i + half < D, P.err, 0x22)) {
                    vp[i] = store1<DT>(a);
                    vp[i + half] = store1<DT>(b);
                }
            }
        }
    }
}

// One (row, kv head) unit of the tick's attention, over the row's whole cache range: thread 0
// streams the K and V rows in chunks of CP positions with bulk copies into the B ring (idle
// between GEMM phases; K in the first half of a slot, V in the second), 4 chunks in flight;
// the 8 worker warps score and accumulate each chunk from shared memory. Query heads
// hoff .. hoff + GC - 1 of the kv head's Gt.
template <int DT, int GC>
__device__ void tick_attn_unit(const KieParams &P, MrShared &S, const AttnArgs &A, int g, int Gt, int hoff,
                               uint32_t &k_it) {
    constexpr int NW = MR_WORKERS / 32, B = 2;
    const int nh = min(GC, Gt - hoff);
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int D = A.D, lpp = D >> 3, ppw = 32 / lpp, sub = lane / lpp, sl = lane % lpp;
    const int ngroups = NW * ppw, gi = w * ppw + sub;  // ngroups * B == CP for every D
    const int rowb = D * 2, CP = (TILE / 2) / rowb;
    const int ctx = A.ctx, nch = (ctx + CP - 1) / CP;
    const uint8_t *kb = reinterpret_cast<const uint8_t *>(A.k + (size_t)g * A.head_stride);
    const uint8_t *vb = reinterpret_cast<const uint8_t *>(A.v + (size_t)g * A.head_stride);
    uint8_t *ring = S.b[0];    // KV_SLOTS chunk slots of TILE bytes over the B ring
    auto issue = [&](int c) {  // chunk c of this unit into its slot (thread 0)
        const uint32_t it = k_it + c, slot = it % KV_SLOTS;
        if (S.abort || !mbar_wait(&S.k_empty[slot], ((it / KV_SLOTS) & 1u) ^ 1u, P.timeout_ns, &S.abort)) {
            if (!S.abort) set_error(P.err, DERR_RING_TIMEOUT, 0x94);
            S.abort = 1;
            return;
        }
        const uint32_t bytes = (uint32_t)(min(CP, ctx - c * CP) * rowb);
        mbar_arrive_expect_tx(&S.k_full[slot], 2 * bytes);
        bulk_g2s(ring + slot * TILE, kb + (size_t)c * CP * rowb, bytes, &S.k_full[slot]);
        bulk_g2s(ring + slot * TILE + TILE / 2, vb + (size_t)c * CP * rowb, bytes, &S.k_full[slot]);
        S.k_iss = it + 1;
    };
    if (tid == 0) {
        fence_proxy_async_global();  // the newest rows were written (generic proxy) before the barrier
        for (int c = 0; c < min(KV_SLOTS, nch); c++) issue(c);
    }
    const float qscale = rsqrtf((float)D) * 1.4426950408889634f;
    float q[GC][8];
#pragma unroll
    for (int jj = 0; jj < GC; jj++) {
        const float *qp = A.q + (size_t)(g * Gt + hoff + min(jj, nh - 1)) * D + sl * 8;
        const float4 a = __ldcg(reinterpret_cast<const float4 *>(qp));
        const float4 b = __ldcg(reinterpret_cast<const float4 *>(qp + 4));
        q[jj][0] = a.x * qscale; q[jj][1] = a.y * qscale; q[jj][2] = a.z * qscale; q[jj][3] = a.w * qscale;
        q[jj][4] = b.x * qscale; q[jj][5] = b.y * qscale; q[jj][6] = b.z * qscale; q[jj][7] = b.w * qscale;
    }
    float m[GC], l[GC], acc[GC][8];
#pragma unroll
    for (int jj = 0; jj < GC; jj++) {
        m[jj] = -CUDART_INF_F;
        l[jj] = 0.f;
#pragma unroll
        for (int e = 0; e < 8; e++) acc[jj][e] = 0.f;
    }
    for (int c = 0; c < nch; c++) {
        const uint32_t it = k_it + c, slot = it % KV_SLOTS;
        const bool ok = __all_sync(0xffffffffu, !S.abort && mbar_wait(&S.k_full[slot], (it / KV_SLOTS) & 1u,
                                                                       P.timeout_ns, &S.abort));
        if (!ok) {
            if (!S.abort) set_error(P.err, DERR_RING_TIMEOUT, 0x95);
            S.abort = 1;
            break;
        }
        uint4 kv[B], vv[B];
#pragma unroll
        for (int b = 0; b < B; b++) {
            const int jl = gi + b * ngroups;
            const bool in = c * CP + jl < ctx;
            kv[b] = in ? *reinterpret_cast<const uint4 *>(ring + slot * TILE + jl * rowb + sl * 16) : make_uint4(0, 0, 0, 0);
            vv[b] = in ? *reinterpret_cast<const uint4 *>(ring + slot * TILE + TILE / 2 + jl * rowb + sl * 16)
                       : make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.k_empty[slot]);  // this warp's reads of the slot are done
        attn_update<DT, GC, B>(kv, vv, c * CP, ctx, gi, ngroups, lpp, q, m, l, acc);
        if (tid == 0 && c + KV_SLOTS < nch) issue(c + KV_SLOTS);
    }
    k_it += nch;
    attn_tail<DT, GC, NW, true>(A, S.at, g, Gt, hoff, m, l, acc);
}

// Tensor-core attention of the tick and of chunked prefill (head_dim a multiple of 64). The
// units (row, kv head) a CTA takes in one attention phase form one stream of 128-position
// tiles, and every tile takes two tcgen05 products:
//   scores  S[p][c] = K[p] . Qt[c]  (M = 128 positions, N = 16, K = head_dim). Columns c < 8
//           hold the 16-bit hi part of the scaled query heads, c >= 8 the lo part, so
//           S[p][h] + S[p][8 + h] is the score of head h to ~16 bits of the fp32 query.
//   values  O[d][c] = sum_p V[p][d] Pt[c][p]  (M = 128 dims, N = 16, K = 128 positions). V is
//           the MN-major operand just as the tile copy lands it; Pt holds p = 2^(s - M) of
//           each head as 16-bit hi (row h) and lo (row 8 + h) parts, so O[d][h] + O[d][8 + h]
//           is the tile's P.V of head h to ~16 bits of p.
// K and V tiles are 2-D TMA copies (no multicast) of 128 positions x 64 dims per box,
// 128-byte swizzled, from tensor maps over the whole K and V arenas, into two stages of the
// weight ring and a third in the activation ring (the producer holds the O weights back until
// attention is done, and no activation tile moves during it). The copies of stream tile k + 3
// -- the next unit's first tiles near the end of a unit -- are issued as soon as tile k's
// products are done, so loads run on across unit boundaries.
// Warp 8 (the GEMM MMA warp, idle in this phase) issues both products of every tile: the
// score product as soon as the tile's K is in and the softmax warps have read the previous
// tile's scores, the P.V once the tile's Pt is written and its V is in. Warps 0-3 run the
// softmax: a position each from TMEM, the running max M per head (the same in every thread)
// and each thread's share of the running sum; they write Pt (two buffers). Warps 4-7 fold
// each tile's P.V (two TMEM buffers) into the output, rescaled by the tile's correction, and
// issue the tile copies. The three roles meet at mbarriers only (one arrival per warp).

// the K and V tile buffers of attention stage st: two stages in the weight ring, one in the
// activation ring (both idle during attention)
KIE_DEV uint8_t *at_kbuf(MrShared &S, int st) { return st < 2 ? S.a[2 * st] : S.b[0]; }
KIE_DEV uint8_t *at_vbuf(MrShared &S, int st) { return st < 2 ? S.a[2 * st + 1] : S.b[1]; }

// thread 0 or 128: the copies of stream tile k (tile k - (tiles of the units before) of its
// unit) into stage st
__device__ void attn_issue(const KieParams &P, MrShared &S, int k, int nunits, int st, int nks) {
    int i = 0;
    while (i < nunits && k >= S.un_nt[i]) k -= S.un_nt[i++];
    if (i >= nunits) return;
    const int y = (int)(S.un_row0[i] + (long long)k * 128);
    mbar_arrive_expect_tx(&S.at_k[st], (uint32_t)(nks * TILE));
    for (int ks = 0; ks < nks; ks++) tma_load_2d(at_kbuf(S, st) + ks * TILE, P.mr_kmap, ks * 64, y, &S.at_k[st]);
    S.tk_iss[st]++;
    mbar_arrive_expect_tx(&S.at_v[st], (uint32_t)(nks * TILE));
    for (int ks = 0; ks < nks; ks++) tma_load_2d(at_vbuf(S, st) + ks * TILE, P.mr_vmap, ks * 64, y, &S.at_v[st]);
    S.tv_iss[st]++;
}

// the score product of the tile in stage st (K tile x query operand) into TMEM
// columns 0-15
KIE_DEV void attn_scores_mma(MrShared &S, const uint8_t *Qt, int st, int nks, uint32_t idesc) {
    // descriptors advance by their start-address field (16-byte units)
    const uint64_t dk = smem_desc_sw128(smem_u32(at_kbuf(S, st))), dq = smem_desc_sw128(smem_u32(Qt));
    const uint32_t tm = S.tmem_base;
#pragma unroll
    for (int ks = 0; ks < 2; ks++) {
        if (ks == nks) break;
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
            umma_f16(tm, dk + (uint64_t)((ks * TILE + kk * 32) >> 4), dq + (uint64_t)((ks * 2048 + kk * 32) >> 4), idesc,
                     (ks | kk) ? 1u : 0u);
    }
    umma_commit(&S.at_s);
}

// the P.V product of the tile in stage st into P.V buffer pb (TMEM columns 32 + 16 pb ..)
KIE_DEV void attn_pv_mma(MrShared &S, const uint8_t *Pt, int st, int pb, uint32_t idesc) {
    const uint32_t tm = S.tmem_base + 32u + 16u * (uint32_t)pb;
    const uint64_t dv = smem_desc_mn_sw128(smem_u32(at_vbuf(S, st))), dp = smem_desc_sw128(smem_u32(Pt));
#pragma unroll
    for (int kb = 0; kb < 2; kb++)
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
            umma_f16(tm, dv + (uint64_t)((kb * 8192 + kk * 2048) >> 4), dp + (uint64_t)((kb * 2048 + kk * 32) >> 4), idesc,
                     (kb | kk) ? 1u : 0u);
    umma_commit(&S.at_o[pb]);
}

// One pass of a unit (row m, kv head g; query heads hoff .. hoff + GC - 1 of its Gt): stream
// entry ui, tiles k0 .. k0 + ntile - 1 of the stream's ktot. Warp 8 issues the products.
template <int DT, int GC>
__device__ void tick_attn_tc(const KieParams &P, MrShared &S, const AttnArgs &A, int g, int Gt, int hoff, int ui,
                             int nunits, int k0, int ktot, unsigned long long &t_it) {
    static_assert(GC <= 8, "the query operand holds 8 heads (hi) + 8 (lo)");
    const int nh = min(GC, Gt - hoff);
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int D = A.D, nks = D >> 6;
    const int ctx = S.un_ctx[ui], ntile = S.un_nt[ui];
    uint8_t *Qt = reinterpret_cast<uint8_t *>(S.at.wacc);  // [nks][16 rows][128 B], swizzled
    uint8_t *Pt0 = Qt + 4096;                              // two tiles of [2][16 rows][128 B], swizzled

    // the query operand: rows h (hi) and 8 + h (lo) of the scaled query heads, other rows zero
    const float qscale = rsqrtf((float)D) * 1.4426950408889634f;
    for (int i = tid; i < 16 * (D >> 3); i += MR_WORKERS) {
        const int row = i / (D >> 3), ch = i % (D >> 3), h = row & 7;
        uint32_t pk[4] = {0u, 0u, 0u, 0u};
        if (h < nh) {
            const float *qp = A.q + (size_t)(g * Gt + hoff + h) * D + ch * 8;
            const float4 a = __ldcg(reinterpret_cast<const float4 *>(qp));
            const float4 b = __ldcg(reinterpret_cast<const float4 *>(qp + 4));
            const float v[8] = {a.x * qscale, a.y * qscale, a.z * qscale, a.w * qscale,
                                b.x * qscale, b.y * qscale, b.z * qscale, b.w * qscale};
#pragma unroll
            for (int j = 0; j < 4; j++) {
                uint16_t e0 = store1<DT>(v[2 * j]), e1 = store1<DT>(v[2 * j + 1]);
                if (row >= 8) {
                    e0 = store1<DT>(v[2 * j] - cvt1<DT>(e0));
                    e1 = store1<DT>(v[2 * j + 1] - cvt1<DT>(e1));
                }
                pk[j] = (uint32_t)e0 | ((uint32_t)e1 << 16);
            }
        }
        *reinterpret_cast<uint4 *>(Qt + (ch >> 3) * 2048 + sw128(row, ch & 7)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    fence_proxy_async_smem();  // generic writes of the query tile -> tensor-core reads
    named_bar_sync(1, MR_WORKERS);
    if (tid == 0) mbar_arrive(&S.at_q);  // warp 8 may issue the unit's score products

    if (w < 4) {  // ---- softmax warps
        float M[GC], Ls[GC];
#pragma unroll
        for (int h = 0; h < GC; h++) {
            M[h] = -CUDART_INF_F;
            Ls[h] = 0.f;
        }
        for (int t = 0; t < ntile; t++) {  // uniform control flow: every thread reaches every barrier
            const int st = (int)(t_it % AT_STAGES);                   // this tile's K/V stage
            const uint32_t spar = (uint32_t)(t_it / AT_STAGES) & 1u;  // ... whose barriers complete every third tile
            const int pb = (int)(t_it & 1ull);                        // its Pt, correction, P.V and max buffers
            const uint32_t prev = (uint32_t)((t_it >> 1) + 1) & 1u;   // the buffers' phase of tile t_it - 2
            const int p0 = t * 128, np = min(128, ctx - p0);
            uint8_t *Pt = Pt0 + pb * 4096;
            float *red = S.at.red + pb * 32;
            const bool ok = __all_sync(0xffffffffu, !S.abort && mbar_wait(&S.at_s, (uint32_t)pb, P.timeout_ns, &S.abort));
            float v[16];
            if (ok) {
                tc_fence_after();
                tmem_ld16(S.tmem_base + ((uint32_t)(w * 32) << 16), v);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.at_sf);  // the warp's scores are read: the next tile's product may follow
            const int pw = w * 32 + lane;  // this thread's position in the tile
            float sc[GC];
#pragma unroll
            for (int h = 0; h < GC; h++) sc[h] = (ok && p0 + pw < ctx && h < nh) ? v[h] + v[8 + h] : -CUDART_INF_F;
#pragma unroll
            for (int h = 0; h < GC; h++) {
                const float mx = warp_max(sc[h]);
                if (lane == 0) red[w * 8 + h] = mx;
            }
            named_bar_sync(2, 128);
            float corr[GC];
#pragma unroll
            for (int h = 0; h < GC; h++) {
                const float mt = fmaxf(fmaxf(red[h], red[8 + h]), fmaxf(red[16 + h], red[24 + h]));
                const float mn = fmaxf(M[h], mt);
                corr[h] = rescale(M[h], mn);
                M[h] = mn;
            }
            // the buffers' last tile (t_it - 2) is folded into the output: Pt, its correction and
            // its P.V accumulator are free
            if (t_it >= 2 && !__all_sync(0xffffffffu, !S.abort && mbar_wait(&S.at_of[pb], prev, P.timeout_ns, &S.abort))) {
                if (lane == 0 && !S.abort) set_error(P.err, DERR_RING_TIMEOUT, 0x99);
                if (lane == 0) S.abort = 1;
            }
#pragma unroll
            for (int h = 0; h < GC; h++)
                if (tid == h) S.at_corr[pb][h] = corr[h];
            // Pt: this position's p of every head, hi in row h and lo in row 8 + h; even lanes
            // store the pair (position, position + 1)
            const int kb = pw >> 6, ch = (pw >> 3) & 7, within = (pw & 7) * 2;
#pragma unroll
            for (int h = 0; h < GC; h++) {
                const float p = rescale(sc[h], M[h]);
                Ls[h] = Ls[h] * corr[h] + p;
                const uint32_t hi = store1<DT>(p), lo = store1<DT>(p - cvt1<DT>((uint16_t)hi));
                const uint32_t hi1 = __shfl_down_sync(0xffffffffu, hi, 1), lo1 = __shfl_down_sync(0xffffffffu, lo, 1);
                if (!(lane & 1)) {
                    *reinterpret_cast<uint32_t *>(Pt + kb * 2048 + sw128(h, ch) + within) = hi | (hi1 << 16);
                    *reinterpret_cast<uint32_t *>(Pt + kb * 2048 + sw128(8 + h, ch) + within) = lo | (lo1 << 16);
                }
            }
            if (np < 128) {  // the last tile: V rows past the context (other positions' data) become zeros
                const bool vok = __all_sync(0xffffffffu, !S.abort && mbar_wait(&S.at_v[st], spar, P.timeout_ns, &S.abort));
                if (vok) {
                    uint8_t *Vs = at_vbuf(S, st);
                    const int per = (128 - np) * 8;  // 16-byte pieces per box
                    for (int i = tid; i < nks * per; i += 128) {
                        const int ks = i / per, r = np + (i % per) / 8, c = i % 8;
                        *reinterpret_cast<uint4 *>(Vs + ks * TILE + r * 128 + c * 16) = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
            }
            fence_proxy_async_smem();  // Pt (and the zeroed V rows) -> tensor-core reads
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.at_p[pb]);  // the warp's part of Pt (and the correction) is in
            t_it++;
        }
#pragma unroll
        for (int h = 0; h < GC; h++) {
            const float s = warp_sum(Ls[h]);
            if (lane == 0) S.at_l[w][h] = s;
        }
        named_bar_sync(1, MR_WORKERS);  // the sums' shares are in
        named_bar_sync(1, MR_WORKERS);  // the unit's output is written
    } else {  // ---- output warps
        const int wq = w - 4;
        float acc[GC];
#pragma unroll
        for (int h = 0; h < GC; h++) acc[h] = 0.f;
        for (int t = 0; t < ntile; t++) {
            const int st = (int)(t_it % AT_STAGES), pb = (int)(t_it & 1ull);
            const uint32_t ph = (uint32_t)(t_it >> 1) & 1u;  // the buffer's barriers complete every other tile
            bool ok = __all_sync(0xffffffffu, !S.abort && mbar_wait(&S.at_p[pb], ph, P.timeout_ns, &S.abort));
            ok = ok && __all_sync(0xffffffffu, !S.abort && mbar_wait(&S.at_o[pb], ph, P.timeout_ns, &S.abort));
            float corr[GC], v[16];
#pragma unroll
            for (int h = 0; h < GC; h++) corr[h] = S.at_corr[pb][h];
            if (ok) {
                tc_fence_after();
                tmem_ld16(S.tmem_base + 32u + 16u * (uint32_t)pb + ((uint32_t)(wq * 32) << 16), v);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.at_of[pb]);  // the warp has read the product and the correction
            if (ok) {
#pragma unroll
                for (int h = 0; h < GC; h++) acc[h] = acc[h] * corr[h] + (v[h] + v[8 + h]);
            }
            // the tile's K and V are consumed: its stage takes stream tile k + AT_STAGES
            if (tid == 128 && !S.abort && k0 + t + AT_STAGES < ktot) {
                fence_proxy_async_smem();
                attn_issue(P, S, k0 + t + AT_STAGES, nunits, st, nks);
            }
            t_it++;
        }
        named_bar_sync(1, MR_WORKERS);  // the sums' shares are in
        const int d = wq * 32 + lane;   // this thread's output dim
#pragma unroll
        for (int h = 0; h < GC; h++) {
            const float L = ((S.at_l[0][h] + S.at_l[1][h]) + S.at_l[2][h]) + S.at_l[3][h];
            const float o = acc[h] / L;
            const float o1 = __shfl_down_sync(0xffffffffu, o, 1);
            if (h < nh && d < D && !(lane & 1) &&
                in_bounds(A.brow < MAXR && (g * Gt + hoff + h) * D + d + 1 < P.Hq * P.D, P.err, 0x28))
                attn_out2<DT>(A, (g * Gt + hoff + h) * D + d, o, o1);
        }
        named_bar_sync(1, MR_WORKERS);  // the unit's output is written
    }
}

// Lane 0 of warp 8: the products of the tensor-core attention of one layer-step, in the order
// the worker warps consume them: the score product of tile k as soon as its K tile is in and
// the softmax threads have read tile k - 1's scores; the P.V of tile k once its Pt is written
// (which also means the output threads are done with the buffer's tile k - 2) and its V is in.
__device__ bool mr_attn_mma(const KieParams &P, MrShared &S, int M, unsigned long long &at_it, uint32_t &q_it,
                            uint32_t &tab_it) {
    const int nks = P.D >> 6;
    const uint32_t idesc_s = idesc_f16(P.dtype, 16), idesc_o = idesc_s | (1u << 15);  // V MN-major
    const uint8_t *Qt = reinterpret_cast<const uint8_t *>(S.at.wacc), *Pt0 = Qt + 4096;
    (void)M;
    for (bool more = true; more;) {  // the worker warps hand over one stream table at a time
        if (!mbar_wait(&S.at_tab, tab_it & 1u, P.timeout_ns, &S.abort)) return false;
        tab_it++;
        const int nb = S.un_n;
        more = S.un_more != 0;
        for (int i = 0; i < nb; i++) {
            const int ntile = S.un_nt[i];
            if (!mbar_wait(&S.at_q, q_it & 1u, P.timeout_ns, &S.abort)) return false;
            q_it++;
            for (int t = 0; t <= ntile; t++) {
                if (t < ntile) {
                    const unsigned long long k = at_it + t;
                    if (!mbar_wait(&S.at_k[k % AT_STAGES], (uint32_t)(k / AT_STAGES) & 1u, P.timeout_ns, &S.abort) ||
                        (k > 0 && !mbar_wait(&S.at_sf, (uint32_t)((k - 1) & 1ull), P.timeout_ns, &S.abort)))
                        return false;
                    tc_fence_after();
                    attn_scores_mma(S, Qt, (int)(k % AT_STAGES), nks, idesc_s);
                }
                if (t > 0) {
                    const unsigned long long k = at_it + t - 1;
                    const int pb = (int)(k & 1ull);
                    if (!mbar_wait(&S.at_p[pb], (uint32_t)(k >> 1) & 1u, P.timeout_ns, &S.abort) ||
                        !mbar_wait(&S.at_v[k % AT_STAGES], (uint32_t)(k / AT_STAGES) & 1u, P.timeout_ns, &S.abort))
                        return false;
                    tc_fence_after();
                    attn_pv_mma(S, Pt0 + pb * 4096, (int)(k % AT_STAGES), pb, idesc_o);
                }
            }
            at_it += ntile;
        }
    }
    return true;
}

// Balanced assignment of a step's attention entries (unit, pass of 4 query heads) to the
// CTAs, computed alike in every CTA. With E entries on nblk CTAs, r = E mod nblk CTAs take
// K + 1 = E / nblk + 1 entries and the others K; the entries, sorted by tiles (descending, then
// by index), go largest first to the K-entry CTAs and the r * (K + 1) smallest to the others.
// Within each group they are dealt in rounds of one per CTA, each round to the CTAs in order
// of the tiles they hold so far (fewest first). Positions do not change within a step, so it
// runs at the first layer; S.un_cnt = -1 leaves the entries dealt in turn (more entries than
// it sorts, or loads past its key range).
__device__ void attn_assign(const KieParams &P, MrShared &S, int M) {
    const int tid = threadIdx.x, npass = (P.G + 3) / 4, E = M * P.Hkv * npass, nblk = P.nblk;
    const int ntmax = (P.max_ctx + 127) >> 7;
    if (E > AS_MAX || nblk > 256 || ntmax > 0xFFFF || (long long)ntmax * E >= (1ll << 23) ||
        (E + nblk - 1) / nblk > AS_LIST) {
        if (tid == 0) S.un_cnt = -1;
        named_bar_sync(1, MR_WORKERS);
        return;
    }
    // scratch in the activation ring (idle until the stream's first copies)
    uint32_t *key = reinterpret_cast<uint32_t *>(S.b[0]);  // [ep] (65535 - tiles) << 16 | entry
    uint32_t *ld = key + AS_MAX;                            // [256] tiles so far << 8 | CTA
    int ep = 1;
    while (ep < E) ep <<= 1;
    for (int i = tid; i < ep; i += MR_WORKERS) {
        uint32_t k = 0xFFFFFFFFu;
        if (i < E) {
            const int m = (i / npass) / P.Hkv;
            const int nt = (__ldcg(P.mr_pos + m) + 128) >> 7;
            k = ((uint32_t)(0xFFFF - nt) << 16) | (uint32_t)i;
        }
        key[i] = k;
    }
    if (tid == 0) S.un_cnt = 0;
    auto bitonic = [&](uint32_t *a, int n) {  // ascending; one thread per compared pair
        for (int k = 2; k <= n; k <<= 1)
            for (int j = k >> 1; j > 0; j >>= 1) {
                named_bar_sync(1, MR_WORKERS);
                for (int i = tid; i < n; i += MR_WORKERS) {
                    const int x = i ^ j;
                    if (x > i) {
                        const uint32_t u = a[i], v = a[x];
                        if ((u > v) == ((i & k) == 0)) {
                            a[i] = v;
                            a[x] = u;
                        }
                    }
                }
            }
        named_bar_sync(1, MR_WORKERS);
    };
    bitonic(key, ep);
    // entries [e0, e0 + n * rounds) to CTAs c0 .. c0 + n - 1, one per CTA per round
    auto deal = [&](int e0, int c0, int n, int rounds) {
        for (int i = tid; i < 256; i += MR_WORKERS) ld[i] = i < n ? (uint32_t)(c0 + i) : 0xFFFFFFFFu;
        for (int r = 0; r < rounds; r++) {
            named_bar_sync(1, MR_WORKERS);
            for (int j = tid; j < n; j += MR_WORKERS) {
                const uint32_t k = key[e0 + r * n + j];
                const uint32_t nt = 0xFFFFu - (k >> 16), cta = ld[j] & 0xFFu;
                ld[j] = (((ld[j] >> 8) + nt) << 8) | cta;
                if ((int)cta == (int)blockIdx.x) {
                    S.un_list[r] = (uint16_t)(k & 0xFFFFu);
                    S.un_cnt = r + 1;
                }
            }
            if (r + 1 < rounds) bitonic(ld, 256);
        }
        named_bar_sync(1, MR_WORKERS);
    };
    const int K = E / nblk, r = E % nblk;
    if (K > 0) deal(0, r, nblk - r, K);               // the largest entries, K per CTA
    if (r > 0) deal((nblk - r) * K, 0, r, K + 1);     // the smallest, K + 1 per CTA
}

// Attention of every row (a tick's sessions or a prefill chunk's positions): one unit per
// (row, kv head), the unit's output written into the O projection's B operand.
template <int DT>
__device__ void phase_attn(const KieParams &P, MrShared &S, int l, int M, uint32_t &k_it, unsigned long long &t_it) {
    const int G = P.G;
    if (P.mr_kmap) {  // head_dim a multiple of 64: both products on the tensor cores
        const int tid = threadIdx.x, nks = P.D >> 6, npass = (G + 3) / 4;
        if (l == 0) attn_assign(P, S, M);
        // this CTA's entries (unit, pass over 4 query heads at a time; one pass up to G = 4)
        const bool dealt = S.un_cnt >= 0;
        const int ne = dealt ? S.un_cnt : (M * P.Hkv - (int)blockIdx.x + P.nblk - 1) / P.nblk * npass;
        auto entry = [&](int i, int &u, int &hoff) {
            const int e = dealt ? (int)S.un_list[i] : ((int)blockIdx.x + (i / npass) * P.nblk) * npass + i % npass;
            u = e / npass;
            hoff = 4 * (e % npass);
        };
        int b0 = 0;
        do {  // streams of up to NU_MAX entries (at least one, maybe empty: warp 8 waits for it)
            const int nb = max(0, min(NU_MAX, ne - b0));
            if (tid < nb) {
                int u, hoff;
                entry(b0 + tid, u, hoff);
                const int m = u / P.Hkv, g = u % P.Hkv;
                const int sid = __ldcg(P.mr_sid + m), pos = __ldcg(P.mr_pos + m);
                S.un_row0[tid] = (((long long)sid * P.L + l) * P.Hkv + g) * P.max_ctx;
                S.un_ctx[tid] = pos + 1;
                S.un_nt[tid] = (pos + 128) >> 7;
            }
            if (tid == 0) {
                S.un_n = nb;
                S.un_more = b0 + nb < ne;
            }
            named_bar_sync(1, MR_WORKERS);
            int ktot = 0;
            for (int i = 0; i < nb; i++) ktot += S.un_nt[i];
            if (tid == 0 || tid == 128) fence_proxy_async_global();  // the newest rows (written before the barrier)
            if (tid == 0) {
                if (!S.abort) {
                    fence_proxy_async_smem();  // earlier reads of the ring before the copies refill it
                    for (int k = 0; k < AT_STAGES && k < ktot; k++) attn_issue(P, S, k, nb, (int)((t_it + k) % AT_STAGES), nks);
                }
                mbar_arrive(&S.at_tab);  // warp 8 may read the stream's table
            }
            int k0 = 0;
            for (int i = 0; i < nb; i++) {
                int u, hoff;
                entry(b0 + i, u, hoff);
                const int m = u / P.Hkv, g = u % P.Hkv;
                AttnArgs A;
                A.q = P.mr_q + (size_t)m * P.Hq * P.D;
                A.o = nullptr;
                A.bpack = P.mr_bpack;  // the output is the O projection's B operand, row m
                A.brow = m;
                A.D = P.D;
                tick_attn_tc<DT, 4>(P, S, A, g, G, hoff, i, nb, k0, ktot, t_it);
                k0 += S.un_nt[i];
            }
            b0 += nb;
        } while (b0 < ne);
        return;
    }
    for (int u = blockIdx.x; u < M * P.Hkv; u += P.nblk) {
        const int m = u / P.Hkv, g = u % P.Hkv;
        const int sid = __ldcg(P.mr_sid + m), pos = __ldcg(P.mr_pos + m);
        AttnArgs A;
        A.q = P.mr_q + (size_t)m * P.Hq * P.D;
        A.k = P.kcache + (size_t)sid * P.sess_stride + (size_t)l * P.Hkv * P.max_ctx * P.D;
        A.v = P.vcache + (size_t)sid * P.sess_stride + (size_t)l * P.Hkv * P.max_ctx * P.D;
        A.head_stride = (long long)P.max_ctx * P.D;
        A.part = nullptr;  // one split: the unit's result is final
        A.cnt = nullptr;
        A.o = nullptr;
        A.bpack = P.mr_bpack;  // the output is the O projection's B operand, row m
        A.brow = m;
        A.gout = g;
        A.cnt_target = 0;
        A.oslice = nullptr;
        A.timeout_ns = 0;
        A.err = nullptr;
        A.D = P.D;
        A.Hkv = P.Hkv;
        A.nsplit = 1;
        A.ctx = pos + 1;
        for (int hoff = 0; hoff < G; hoff += 4) tick_attn_unit<DT, 4>(P, S, A, g, G, hoff, k_it);
    }
}

__device__ __forceinline__ void amax(float &v, int &i, float v2, int i2) {
    if (v2 > v || (v2 == v && i2 < i)) {
        v = v2;
        i = i2;
    }
}

// argmax of each row's logits (one CTA per row); outputs and the next step's inputs. The
// row is read as float4 with 8 loads in flight per thread (lowest index wins ties).
__device__ void phase_argmax(const KieParams &P, MrShared &S, const KieCmd &cmd, int step, int M) {
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    for (int m = blockIdx.x; m < M; m += P.nblk) {
        const float *lg = P.mr_logits + (size_t)m * P.V;
        float bv = -CUDART_INF_F;
        int bi = 0x7fffffff;
        const bool copy = cmd.logits && (cmd.op == OP_TICK || m == M - 1);
        float *dst = nullptr;
        if (copy) dst = cmd.logits + (cmd.op == OP_TICK ? ((size_t)step * M + m) * P.V : 0);
        // rows start 16-byte aligned when V % 4 == 0; otherwise take the scalar path
        const int n4 = (P.V % 4 == 0) ? P.V / 4 : 0;
        const float4 *lg4 = reinterpret_cast<const float4 *>(lg);
        const bool dst4 = dst && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0;  // caller's buffer may be unaligned
        for (int r0 = tid; r0 < n4; r0 += MR_WORKERS * 8) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int r = r0 + u * MR_WORKERS;
                v[u] = r < n4 ? __ldcg(lg4 + r) : make_float4(-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F);
            }
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int r = r0 + u * MR_WORKERS;
                if (r < n4) {
                    if (dst4) {
                        reinterpret_cast<float4 *>(dst)[r] = v[u];
                    } else if (dst) {
                        dst[4 * r] = v[u].x;
                        dst[4 * r + 1] = v[u].y;
                        dst[4 * r + 2] = v[u].z;
                        dst[4 * r + 3] = v[u].w;
                    }
                    amax(bv, bi, v[u].x, 4 * r);
                    amax(bv, bi, v[u].y, 4 * r + 1);
                    amax(bv, bi, v[u].z, 4 * r + 2);
                    amax(bv, bi, v[u].w, 4 * r + 3);
                }
            }
        }
        for (int r = 4 * n4 + tid; r < P.V; r += MR_WORKERS) {
            const float v = __ldcg(lg + r);
            if (dst) dst[r] = v;
            amax(bv, bi, v, r);
        }
        for (int o = 16; o > 0; o >>= 1) amax(bv, bi, __shfl_xor_sync(0xffffffffu, bv, o), __shfl_xor_sync(0xffffffffu, bi, o));
        if (lane == 0) {
            S.red[w] = bv;
            S.red[8 + w] = __int_as_float(bi);
        }
        named_bar_sync(1, MR_WORKERS);
        // the session's sampling (the variant beside argmax): top-k of the row's logits, then the
        // draw of the step's position (attention's shared memory is free in this phase)
        const int sid = __ldcg(P.mr_sid + m);
        const int topk = __ldcg(&P.samp[sid].top_k);
        const bool sample = topk > 1 && (cmd.op == OP_TICK || m == M - 1);
        int sampled = 0;
        if (sample) {
            SampleScratch &SS = *reinterpret_cast<SampleScratch *>(&S.at);
            block_topk<MR_WORKERS>(SS, P.V, topk, [&](int p) { return __ldcg(lg + p); }, [&](int p) { return p; });
            if (tid < 32)
                sampled = sample_pick(SS, topk, __ldcg(&P.samp[sid].inv_t),
                                      sample_uniform(__ldcg(&P.samp[sid].seed), __ldcg(P.mr_pos + m)));
        }
        if (tid == 0) {
            float v = S.red[0];
            int i = __float_as_int(S.red[8]);
            for (int k = 1; k < MR_WORKERS / 32; k++) amax(v, i, S.red[k], __float_as_int(S.red[8 + k]));
            if (sample) i = sampled;
            if (i < 0 || i >= P.V) {  // non-finite logits (no index wins): fail the command
                set_error(P.err, DERR_BAD_TOKEN, 0x41);
                S.abort = 1;
            }
            P.mr_tok[m] = i;                          // input of the next step
            P.mr_pos[m] = __ldcg(P.mr_pos + m) + 1;
            if (cmd.out) {
                if (cmd.op == OP_TICK) cmd.out[step * M + m] = i;
                else if (m == M - 1) cmd.out[0] = i;
            }
        }
        named_bar_sync(1, MR_WORKERS);
    }
}

// ------------------------------------------------------------------ one command, workers' view

// a GEMM phase from the workers' side: thread 0 streams the B tiles, warps 4-7 drain TMEM
__device__ __forceinline__ void mr_gemm(const KieParams &P, MrShared &S, uint32_t &b_it, uint32_t &u_it, int g, int M) {
    if (threadIdx.x < 32) {
        if (threadIdx.x == 0) mr_bload(P, S, b_it, g);
        __syncwarp();  // warp 0 converges again before the grid barrier's bar.sync
    } else if (threadIdx.x >= 128) {
        mr_epilogue(P, S, u_it, g, M);
    }
}

// phase trace (thread 0 of each CTA; same record layout as the batch-1 kernel, one record per
// step of the command)
__device__ __forceinline__ void mr_mark(const KieParams &P, int st, int ev) {
    if (P.trace && st < P.trace_tokens && threadIdx.x == 0)
        P.trace[((size_t)blockIdx.x * P.trace_tokens + st) * P.trace_events + ev] = globaltimer();
}

template <int DT>
__device__ void mr_work(const KieParams &P, MrShared &S, uint32_t &b_it, uint32_t &u_it, uint32_t &k_it,
                        unsigned long long &t_it, const KieCmd &cmd, unsigned long long &epoch) {
    const int M = cmd.n_sess;
    const int steps = steps_of(cmd);
    for (int st = 0; st < steps; st++) {
        mr_mark(P, st, 0);
        for (int l = 0; l < P.L; l++) {
            const int e = 1 + 16 * l;
            if (!S.abort) phase_norm<DT>(P, S, G_QKV, l, l == 0, M);
            mr_mark(P, st, e);
            mr_barrier(P, S, epoch, P.timeout_ns, 1);
            mr_mark(P, st, e + 1);
            mr_gemm(P, S, b_it, u_it, G_QKV, M);
            mr_barrier(P, S, epoch, P.timeout_ns, 2);
            mr_mark(P, st, e + 3);
            if (!S.abort) phase_rope<DT>(P, l, M);
            mr_barrier(P, S, epoch, P.timeout_ns, 3);
            mr_mark(P, st, e + 4);
            if (!S.abort) phase_attn<DT>(P, S, l, M, k_it, t_it);
            named_bar_sync(1, MR_WORKERS);  // every worker is done with the ring
            if (threadIdx.x == 0) {
                __threadfence_block();
                S.att_seq = S.att_seq + 1;  // the producer may now fill the ring with the O weights
            }
            mr_mark(P, st, e + 5);
            mr_barrier(P, S, epoch, P.timeout_ns, 4);
            mr_mark(P, st, e + 6);
            mr_gemm(P, S, b_it, u_it, G_O, M);
            mr_barrier(P, S, epoch, P.timeout_ns, 5);
            mr_mark(P, st, e + 7);
            if (!S.abort) phase_norm<DT>(P, S, G_GU, l, false, M);
            mr_barrier(P, S, epoch, P.timeout_ns, 6);
            mr_mark(P, st, e + 8);
            mr_gemm(P, S, b_it, u_it, G_GU, M);
            mr_barrier(P, S, epoch, P.timeout_ns, 7);
            mr_mark(P, st, e + 9);
            if (!S.abort) phase_act<DT>(P, M);
            mr_barrier(P, S, epoch, P.timeout_ns, 12);
            mr_mark(P, st, e + 10);
            mr_gemm(P, S, b_it, u_it, G_DOWN, M);
            mr_barrier(P, S, epoch, P.timeout_ns, 8);
            mr_mark(P, st, e + 11);
        }
        if (head_needed(cmd)) {
            const int eh = 1 + 16 * P.L;
            if (!S.abort) phase_norm<DT>(P, S, G_HEAD, P.L, false, M);
            mr_barrier(P, S, epoch, P.timeout_ns, 9);
            mr_mark(P, st, eh);
            mr_gemm(P, S, b_it, u_it, G_HEAD, M);
            mr_barrier(P, S, epoch, P.timeout_ns, 10);
            mr_mark(P, st, eh + 1);
            if (!S.abort) phase_argmax(P, S, cmd, st, M);
            mr_barrier(P, S, epoch, P.timeout_ns, 11);
            mr_mark(P, st, eh + 2);
        }
    }
}

// ------------------------------------------------------------------ the kernel

template <int DT>
__global__ void __launch_bounds__(MR_THREADS, 1) kie_mr_kernel(KieParams P, KieCmd one, int resident) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // the swizzled MMA operands need 1024-byte aligned tiles: align the base by hand
    const uint32_t mis = smem_u32(smem_raw) & 1023u;
    MrShared &S = *reinterpret_cast<MrShared *>(smem_raw + ((1024u - mis) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        for (int i = 0; i < A_SLOTS; i++) {
            mbar_init(&S.a_full[i], 1);
            mbar_init(&S.a_empty[i], 1);
        }
        for (int i = 0; i < B_SLOTS; i++) {
            mbar_init(&S.b_full[i], 1);
            mbar_init(&S.b_empty[i], 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&S.acc_full[i], 1);
            mbar_init(&S.acc_empty[i], 4);
        }
        mbar_init(&S.drain, 1);
        for (int i = 0; i < KV_SLOTS; i++) {
            mbar_init(&S.k_full[i], 1);
            mbar_init(&S.k_empty[i], MR_WORKERS / 32);
        }
        S.k_iss = 0;
        for (int i = 0; i < AT_STAGES; i++) {
            mbar_init(&S.at_k[i], 1);
            mbar_init(&S.at_v[i], 1);
            S.tk_iss[i] = S.tv_iss[i] = 0;
        }
        mbar_init(&S.at_s, 1);
        mbar_init(&S.at_sf, 4);  // one arrival per softmax warp
        for (int i = 0; i < 2; i++) {
            mbar_init(&S.at_p[i], 4);
            mbar_init(&S.at_o[i], 1);
            mbar_init(&S.at_of[i], 4);  // one arrival per output warp
        }
        mbar_init(&S.at_q, 1);
        mbar_init(&S.at_tab, 1);
        S.att_seq = 0;
        fence_mbar_init();
        S.abort = 0;
    }
    if (tid < NG) {
        S.a0[tid] = P.mr_a0[tid * (P.nblk + 1) + blockIdx.x];
        S.a1[tid] = P.mr_a0[tid * (P.nblk + 1) + blockIdx.x + 1];
    }
    if (warp == 8) {
        tmem_alloc(&S.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    uint32_t a_it = 0, b_it = 0, u_it = 0, k_it = 0, o_seq = 0, drains = 0, q_it = 0, tab_it = 0;
    unsigned long long t_it = 0;  // attention tiles so far (stage = t_it mod 3 never jumps at a wrap)
    unsigned long long epoch = 0;
    for (;;) {
        if (tid < MR_WORKERS) {
            if (!resident) {
                if (tid == 0) S.cmd = one;
            } else {
                if (blockIdx.x == 0) {
                    if (tid == 0) {
                        const unsigned last = *P.last_seq;
                        const uint64_t t0 = globaltimer();
                        KieCmd c{};
                        c.op = OP_EXIT;
                        for (;;) {
                            const uint32_t s = ld_acquire_sys_u32(&P.mbox->cmd_seq);
                            if (s != last) {
                                copy_cmd(&c, &P.mbox->cmd, true);
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
                    named_bar_sync(1, MR_WORKERS);
                    // rows of the command arrive in the mailbox: sessions, positions, tokens
                    if (S.cmd.op == OP_TICK || S.cmd.op == OP_PREFILL) {
                        const volatile int32_t *io = (const volatile int32_t *)S.cmd.tokens;
                        for (int m = tid; m < S.cmd.n_sess; m += MR_WORKERS) {
                            P.mr_sid[m] = io[m];
                            P.mr_pos[m] = io[MAXR + m];
                            P.mr_tok[m] = io[2 * MAXR + m];
                        }
                    }
                }
                mr_barrier(P, S, epoch, P.idle_ns + P.timeout_ns, 0);
                if (tid == 0) {
                    copy_cmd(&S.cmd, P.cmd, false);
                    if (S.abort) S.cmd.op = OP_EXIT;
                }
            }
        }
        __syncthreads();
        const KieCmd cmd = S.cmd;
        if (cmd.op != OP_TICK && cmd.op != OP_PREFILL) break;
        if (warp == 9) {
            if ((tid & 31) == 0) mr_produce(P, S, a_it, o_seq, cmd);
        } else if (warp == 8) {
            if ((tid & 31) == 0) {
                mr_mma(P, S, a_it, b_it, u_it, t_it, q_it, tab_it, cmd);
                mbar_wait(&S.drain, drains & 1u, P.timeout_ns, nullptr);
            }
            drains++;
        } else {
            mr_work<DT>(P, S, b_it, u_it, k_it, t_it, cmd, epoch);
            if (tid == 0) {  // copies still in flight (only after an abort) land before the CTA moves on
                const uint32_t first = b_it > B_SLOTS ? b_it - B_SLOTS : 0;
                for (uint32_t k = first; k < b_it; k++)
                    mbar_wait(&S.b_full[k % B_SLOTS], (k / B_SLOTS) & 1u, P.timeout_ns, nullptr);
                const uint32_t kfirst = S.k_iss > KV_SLOTS ? S.k_iss - KV_SLOTS : 0;
                for (uint32_t k = kfirst; k < S.k_iss; k++)
                    mbar_wait(&S.k_full[k % KV_SLOTS], (k / KV_SLOTS) & 1u, P.timeout_ns, nullptr);
                // the tensor-core attention's last K, V loads (its products drain with warp 8's)
                for (int i = 0; i < AT_STAGES; i++) {  // per stage: its k-th copy completes phase k - 1
                    if (S.tk_iss[i]) mbar_wait(&S.at_k[i], (S.tk_iss[i] - 1) & 1u, P.timeout_ns, nullptr);
                    if (S.tv_iss[i]) mbar_wait(&S.at_v[i], (S.tv_iss[i] - 1) & 1u, P.timeout_ns, nullptr);
                }
            }
        }
        __syncthreads();
        if (resident && blockIdx.x == 0 && tid == 0) {
            __threadfence_system();
            P.mbox->status = S.abort ? -1 : 0;
            st_release_sys_u32(&P.mbox->done_seq, cmd.seq);
        }
        if (!resident || S.abort) break;
    }
    // release TMEM (warp 8 allocated it; every MMA has drained)
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(S.tmem_base, TMEM_COLS);
    }
}

}  // namespace

// ------------------------------------------------------------------ host-side launch helpers

extern "C++" {

size_t kie_mr_smem_bytes() { return sizeof(MrShared) + 1024; }

cudaError_t kie_mr_prepare(int dtype) {
    const int smem = (int)kie_mr_smem_bytes();
    return dtype == KIE_BF16
               ? cudaFuncSetAttribute(kie_mr_kernel<KIE_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)
               : cudaFuncSetAttribute(kie_mr_kernel<KIE_FP16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

cudaError_t kie_mr_occupancy(int dtype, int *blocks_per_sm) {
    const size_t smem = kie_mr_smem_bytes();
    return dtype == KIE_BF16
               ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, kie_mr_kernel<KIE_BF16>, MR_THREADS, smem)
               : cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, kie_mr_kernel<KIE_FP16>, MR_THREADS, smem);
}

cudaError_t kie_mr_launch(const KieParams &P, const KieCmd &one, int resident, cudaStream_t stream) {
    KieParams p = P;
    KieCmd c = one;
    int r = resident;
    void *args[] = {&p, &c, &r};
    const void *fn = P.dtype == KIE_BF16 ? (const void *)kie_mr_kernel<KIE_BF16> : (const void *)kie_mr_kernel<KIE_FP16>;
    return cudaLaunchCooperativeKernel(fn, dim3(P.nblk), dim3(MR_THREADS), args, kie_mr_smem_bytes(), stream);
}

// Swizzled 128 x 64 tile image of rows [128 rb, 128 rb + 128) and columns [64 ks, 64 ks + 64) of
// a row-major [N][K] matrix that is the row concatenation of up to three row-major parts
// (rows [0, n0) from src[0], [n0, n1) from src[1], [n1, N) from src[2]); rows past N are
// zero. The repack kernel below writes it.
struct TileSrc {
    const uint8_t *src[3];
    long long dst;
    int n0, n1, N, K, rb, ks;
};

__global__ void mr_repack_kernel(const TileSrc *t, long long n, uint8_t *arena) {
    for (long long i = blockIdx.x; i < n; i += gridDim.x) {
        const TileSrc s = t[i];
        for (int c16 = threadIdx.x; c16 < 128 * 8; c16 += blockDim.x) {
            const int r = c16 >> 3, c = c16 & 7;
            const int row = s.rb * 128 + r;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (row < s.N) {
                const int part = row < s.n0 ? 0 : row < s.n1 ? 1 : 2;
                const int prow = row - (part == 0 ? 0 : part == 1 ? s.n0 : s.n1);
                v = *reinterpret_cast<const uint4 *>(s.src[part] + ((size_t)prow * s.K + s.ks * 64 + c * 8) * 2);
            }
            *reinterpret_cast<uint4 *>(arena + s.dst + r * 128 + ((c ^ (r & 7)) << 4)) = v;
        }
    }
}

cudaError_t kie_mr_repack(const void *tiles, long long n, uint8_t *arena, cudaStream_t stream) {
    mr_repack_kernel<<<1184, 256, 0, stream>>>(static_cast<const TileSrc *>(tiles), n, arena);
    return cudaGetLastError();
}

size_t kie_mr_tile_src_bytes() { return sizeof(TileSrc); }

void kie_mr_tile_src(void *dst, const void *const *src3, int n0, int n1, long long off, int N, int K, int rb, int ks) {
    TileSrc t;
    for (int i = 0; i < 3; i++) t.src[i] = static_cast<const uint8_t *>(src3[i]);
    t.dst = off;
    t.n0 = n0;
    t.n1 = n1;
    t.N = N;
    t.K = K;
    t.rb = rb;
    t.ks = ks;
    *static_cast<TileSrc *>(dst) = t;
}

}  // extern "C++"
