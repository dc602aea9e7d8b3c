// Host side of the decode engine: validation, the fixed (ahead-of-time) schedule and
// memory layout, the weight repack, sessions, the doorbell and kernel launches.
//
// Everything the kernels will touch is allocated in kie_create and laid out once: the
// schedule and addresses are fixed before the first token, with no allocator or scheduler
// at run time ("实时AI推理为何贵56倍？…", section 把一切提前决定好). Per call the host only
// writes input tokens into a mapped mailbox and reads output tokens back (same page,
// section 让工作常驻 GPU).
#include <cuda.h>
#include <cuda_runtime.h>
#include <emmintrin.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "kie_internal.h"

// kernels of the other translation units
size_t kie_b1_smem_bytes();
int kie_b1_chunk_rows(int K);
int kie_b1_max_rows(int K);
bool kie_b1_tmem_ok(int d, bool f8);
cudaError_t kie_b1_prepare(int dtype, bool f8, bool tm, bool kvr);
cudaError_t kie_b1_occupancy(int dtype, bool f8, bool tm, bool kvr, int *blocks_per_sm);
cudaError_t kie_b1_launch(const KieParams &P, const KieCmd &one, int resident, cudaStream_t stream);
size_t kie_mr_smem_bytes();
cudaError_t kie_mr_prepare(int dtype);
cudaError_t kie_mr_occupancy(int dtype, int *blocks_per_sm);
cudaError_t kie_mr_launch(const KieParams &P, const KieCmd &one, int resident, cudaStream_t stream);
cudaError_t kie_mr_repack(const void *tiles, long long n, uint8_t *arena, cudaStream_t stream);
cudaError_t kie_fp8_quantize(const void *w, long long rows, int cols, int dtype, uint8_t *q, float *scale,
                             cudaStream_t stream);
size_t kie_mr_tile_src_bytes();
void kie_mr_tile_src(void *dst, const void *const *src3, int n0, int n1, long long off, int N, int K, int rb, int ks);

namespace {

struct RowCopy {
    long long dst;
    const uint8_t *src;
    long long bytes;
};

__global__ void gather_rows_kernel(const RowCopy *rc, long long n, uint8_t *arena) {
    for (long long i = blockIdx.x; i < n; i += gridDim.x) {
        const RowCopy r = rc[i];
        for (long long b = (long long)threadIdx.x * 16; b < r.bytes; b += (long long)blockDim.x * 16)
            *reinterpret_cast<uint4 *>(arena + r.dst + b) = *reinterpret_cast<const uint4 *>(r.src + b);
    }
}

// One fold block of the batch-1 stream: columns [col0, col0 + 8 ng) of a row-major matrix with
// rows of `ld` bytes, written as [ng][rows][8] (16 bytes per row and column group).
struct FoldCopy {
    long long dst;
    const uint8_t *src;
    long long ld;
    int col0, ng, rows, esz;  // esz: bytes per element (2, or 1 for E4M3 codes)
};

__global__ void fold_pack_kernel(const FoldCopy *fc, long long n, uint8_t *arena) {
    for (long long i = blockIdx.x; i < n; i += gridDim.x) {
        const FoldCopy f = fc[i];
        const long long vecs = (long long)f.ng * f.rows;
        for (long long v = threadIdx.x; v < vecs; v += blockDim.x) {
            const long long g = v / f.rows, r = v % f.rows;
            const uint8_t *src = f.src + r * f.ld + (long long)(f.col0 + 8 * g) * f.esz;
            if (f.esz == 2) *reinterpret_cast<uint4 *>(arena + f.dst + v * 16) = *reinterpret_cast<const uint4 *>(src);
            else *reinterpret_cast<uint2 *>(arena + f.dst + v * 8) = *reinterpret_cast<const uint2 *>(src);
        }
    }
}

enum { KIND_NONE = 0, KIND_B1 = 1, KIND_MR = 2 };

double now_s() {
    return std::chrono::duration<double>(std::chrono::steady_clock::now().time_since_epoch()).count();
}

}  // namespace

struct kie_engine {
    kie_config cfg{};
    int dev = 0, nblk = 0;
    KieParams P{};
    std::vector<void *> dev_allocs;
    KieMailbox *mbox_host = nullptr;
    KieMailbox *mbox_dev = nullptr;
    int64_t io_ints = 0;
    cudaStream_t stream = nullptr;
    cudaEvent_t ev_done = nullptr;
    int resident = KIND_NONE;  // which kernel currently sits resident on the GPU
    uint32_t seq = 0;
    std::vector<int> sess_len;
    std::vector<char> sess_used;
    bool poisoned = false;
    int pending_fault = KIE_FAULT_NONE;  // kie_inject_fault: applied to the next kernel launch
    std::string err;

    // Clears the grid-barrier counter before a launch. With KIE_FAULT_BARRIER_SHORT pending it
    // starts one arrival short instead (all ones: the first arrival wraps it to zero, so after
    // every CTA has arrived it reads nblk - 1), and the first grid barrier of the launch cannot
    // complete.
    cudaError_t reset_barrier(cudaStream_t st) {
        const int fill = pending_fault == KIE_FAULT_BARRIER_SHORT ? 0xFF : 0;
        pending_fault = KIE_FAULT_NONE;
        cudaError_t e = cudaMemsetAsync(P.bar, fill, 16, st);
        return e == cudaSuccess ? cudaMemsetAsync(P.rd, 0, 8, st) : e;
    }

    kie_status fail(kie_status s, const char *fmt, ...) {
        char buf[512];
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(buf, sizeof buf, fmt, ap);
        va_end(ap);
        err = buf;
        if (s == KIE_ERR_TIMEOUT || s == KIE_ERR_DEVICE) poisoned = true;
        return s;
    }
    kie_status cuda_fail(cudaError_t e, const char *what) {
        return fail(KIE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    }
#ifdef KIE_CHECK_BOUNDS
    // Diagnostic build: every engine buffer sits between two guard regions of GUARD bytes
    // filled with GUARD_BYTE; check_guards() reports any that a kernel (or anyone) overwrote.
    static constexpr size_t GUARD = 256;
    static constexpr int GUARD_BYTE = 0xA5;
    std::vector<std::pair<uint8_t *, size_t>> guarded;  // user region, its bytes
    template <class T>
    cudaError_t alloc(T **p, size_t bytes) {
        bytes = bytes < 16 ? 16 : bytes;
        uint8_t *q = nullptr;
        cudaError_t e = cudaMalloc(&q, bytes + 2 * GUARD);
        if (e != cudaSuccess) return e;
        dev_allocs.push_back(q);
        e = cudaMemset(q, GUARD_BYTE, GUARD);
        if (e == cudaSuccess) e = cudaMemset(q + GUARD + bytes, GUARD_BYTE, GUARD);
        guarded.push_back({q + GUARD, bytes});
        *p = reinterpret_cast<T *>(q + GUARD);
        return e;
    }
    // index of the first buffer whose guard words changed, or -1
    int check_guards() const {
        std::vector<uint8_t> h(GUARD);
        for (size_t i = 0; i < guarded.size(); i++) {
            for (int side = 0; side < 2; side++) {
                const uint8_t *g = side ? guarded[i].first + guarded[i].second : guarded[i].first - GUARD;
                if (cudaMemcpy(h.data(), g, GUARD, cudaMemcpyDeviceToHost) != cudaSuccess) return (int)i;
                for (uint8_t b : h)
                    if (b != GUARD_BYTE) return (int)i;
            }
        }
        return -1;
    }
#else
    template <class T>
    cudaError_t alloc(T **p, size_t bytes) {
        void *q = nullptr;
        cudaError_t e = cudaMalloc(&q, bytes < 16 ? 16 : bytes);
        if (e == cudaSuccess) {
            dev_allocs.push_back(q);
            *p = static_cast<T *>(q);
        }
        return e;
    }
#endif
};

#define CK(expr, what)                                        \
    do {                                                      \
        cudaError_t _e = (expr);                              \
        if (_e != cudaSuccess) return eng->cuda_fail(_e, what); \
    } while (0)

// ---------------------------------------------------------------- small C-ABI helpers

extern "C" void kie_config_defaults(kie_config *c) {
    if (!c) return;
    memset(c, 0, sizeof *c);
    c->rms_eps = 1e-5f;
    c->rope_theta = 1e4f;
    c->dtype = KIE_FP16;
    c->max_sessions = 1;
    c->max_ctx = 4096;
    c->timeout_ms = 10000;
    c->idle_ms = 200;
    c->modes = KIE_MODE_BATCH1;
    c->device = 0;
}

extern "C" const char *kie_status_string(kie_status s) {
    switch (s) {
        case KIE_OK: return "ok";
        case KIE_ERR_ARG: return "bad argument";
        case KIE_ERR_CAPACITY: return "capacity exceeded";
        case KIE_ERR_CUDA: return "CUDA error";
        case KIE_ERR_TIMEOUT: return "timeout";
        case KIE_ERR_STATE: return "engine poisoned";
        case KIE_ERR_DEVICE: return "device error";
        case KIE_ERR_UNSUPPORTED: return "mode not enabled";
        default: return "unknown status";
    }
}

extern "C" kie_status kie_last_error(kie_engine *eng, char *buf, int32_t len) {
    if (!eng || !buf || len <= 0) return KIE_ERR_ARG;
    snprintf(buf, (size_t)len, "%s", eng->err.c_str());
    return KIE_OK;
}

// ---------------------------------------------------------------- validation and plan

static const char *shape_error(const kie_config &c) {
    if (c.n_layers <= 0 || c.d_model <= 0 || c.n_heads <= 0 || c.n_kv_heads <= 0 || c.head_dim <= 0 || c.ffn <= 0 ||
        c.vocab <= 0)
        return "all shape fields must be positive";
    if (c.dtype != KIE_FP16 && c.dtype != KIE_BF16) return "dtype must be KIE_FP16 or KIE_BF16";
    if (c.d_model % 64 || (c.n_heads * c.head_dim) % 64 || c.ffn % 64)
        return "d_model, n_heads*head_dim and ffn must be multiples of 64";
    if (c.head_dim != 8 && c.head_dim != 16 && c.head_dim != 32 && c.head_dim != 64 && c.head_dim != 128)
        return "head_dim must be 8, 16, 32, 64 or 128";
    if (c.n_heads % c.n_kv_heads || c.n_heads / c.n_kv_heads > KIE_GMAX)
        return "n_heads must be a multiple of n_kv_heads, at most 8 query heads per kv head";
    if (c.d_model > 8192) return "d_model above 8192 is not supported";
    if (c.ffn > 14336 || c.n_heads * c.head_dim > 14336) return "ffn and n_heads*head_dim must be <= 14336";
    if ((c.ffn > 8192 && c.ffn % 128) || (c.n_heads * c.head_dim > 8192 && (c.n_heads * c.head_dim) % 128))
        return "ffn and n_heads*head_dim above 8192 must be multiples of 128";
    if (c.max_sessions <= 0 || c.max_ctx <= 0) return "max_sessions and max_ctx must be positive";
    if (c.timeout_ms <= 0 || c.idle_ms <= 0) return "timeouts must be positive";
    if (!(c.modes & (KIE_MODE_BATCH1 | KIE_MODE_TICK))) return "modes must enable at least one kernel";
    if (c.weight_fp8 != 0 && (c.weight_fp8 != 1 || c.modes != KIE_MODE_BATCH1))
        return "weight_fp8 must be 0 or 1, and 1 needs modes == KIE_MODE_BATCH1";
    if (c.b1_staging != 0 && c.b1_staging != 1) return "b1_staging must be 0 or 1";
    if (c.b1_kv_path < 0 || c.b1_kv_path > 2) return "b1_kv_path must be 0, 1 or 2";
    return nullptr;
}

// Units [c*n/nblk, (c+1)*n/nblk) of `unit` rows each.
static void partition(int *row0, int n_units, int unit, int nblk) {
    for (int c = 0; c <= nblk; c++) row0[c] = (int)((long long)c * n_units / nblk) * unit;
}

// Logical row r of the QKV phase (rotation pairs (i, i + D/2) adjacent, v rows paired the same
// way): its matrix (1 = wq, 2 = wk, 3 = wv in a layer's weight list) and row in that matrix.
static void qkv_row(const kie_config &c, int r, int *mat, int *row) {
    const int D = c.head_dim, qd = c.n_heads * D, kvd = c.n_kv_heads * D;
    const int j = r % D, dim = (j >> 1) + (j & 1) * (D >> 1);
    int head;
    if (r < qd) { *mat = 1; head = r / D; }
    else if (r < qd + kvd) { *mat = 2; head = (r - qd) / D; }
    else { *mat = 3; head = (r - qd - kvd) / D; }
    *row = head * D + dim;
}

extern "C" kie_status kie_create(const kie_config *cfg, const kie_weights *w, kie_engine **out) {
    if (!out) return KIE_ERR_ARG;
    *out = nullptr;
    if (!cfg || !w || !w->tok_emb || !w->layers || !w->final_norm || !w->lm_head) return KIE_ERR_ARG;
    if (shape_error(*cfg)) return KIE_ERR_ARG;
    kie_engine *eng = new kie_engine();
    eng->cfg = *cfg;
    const kie_config &c = eng->cfg;
    auto bail = [&](kie_status s) {
        kie_destroy(eng);
        return s;
    };
    // a failed CUDA call releases everything allocated so far
#define CKC(expr, what)                                               \
    do {                                                              \
        cudaError_t _e = (expr);                                      \
        if (_e != cudaSuccess) return bail(eng->cuda_fail(_e, what)); \
    } while (0)
    const bool b1 = (c.modes & KIE_MODE_BATCH1) != 0, mr = (c.modes & KIE_MODE_TICK) != 0;
    cudaError_t e = cudaSetDevice(c.device);
    if (e != cudaSuccess) return bail(eng->cuda_fail(e, "cudaSetDevice"));
    int sms = 0, coop = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, c.device);
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, c.device);
    if (!coop || sms <= 0 || sms > KIE_MAX_CTAS) {
        eng->fail(KIE_ERR_CUDA, "device lacks cooperative launch");
        return bail(KIE_ERR_CUDA);
    }
    // batch-1 weights staged on into TMEM where the kernel's chunk layouts allow it
    const bool b1_tm = c.b1_staging == 1 && kie_b1_tmem_ok(c.d_model, c.weight_fp8 != 0);
    // the attention's K/V through the weight ring at long contexts, from L2 otherwise
    const bool b1_kvr = c.b1_kv_path == 2 || (c.b1_kv_path == 0 && c.max_ctx > 8192);
    if (b1) {
        e = kie_b1_prepare(c.dtype, c.weight_fp8 != 0, b1_tm, b1_kvr);
        if (e != cudaSuccess) return bail(eng->cuda_fail(e, "kernel attributes"));
        int occ = 0;
        e = kie_b1_occupancy(c.dtype, c.weight_fp8 != 0, b1_tm, b1_kvr, &occ);
        if (e != cudaSuccess || occ < 1)
            return bail(eng->cuda_fail(e == cudaSuccess ? cudaErrorInvalidConfiguration : e,
                                       "batch-1 megakernel does not fit on an SM"));
    }
    if (mr) {
        e = kie_mr_prepare(c.dtype);
        if (e != cudaSuccess) return bail(eng->cuda_fail(e, "kernel attributes"));
        int occ = 0;
        e = kie_mr_occupancy(c.dtype, &occ);
        if (e != cudaSuccess || occ < 1)
            return bail(eng->cuda_fail(e == cudaSuccess ? cudaErrorInvalidConfiguration : e,
                                       "tick megakernel does not fit on an SM"));
    }
    const int nblk = sms;
    eng->nblk = nblk;
    const int L = c.n_layers, d = c.d_model, D = c.head_dim, Hq = c.n_heads, Hkv = c.n_kv_heads, F = c.ffn,
              V = c.vocab;
    const int G = Hq / Hkv, qd = Hq * D, kvd = Hkv * D;
    KieParams &P = eng->P;
    P.L = L; P.d = d; P.Hq = Hq; P.Hkv = Hkv; P.D = D; P.F = F; P.V = V; P.dtype = c.dtype; P.G = G;
    P.eps = c.rms_eps;
    P.max_ctx = c.max_ctx;
    P.max_sessions = c.max_sessions;
    P.nblk = nblk;
    P.timeout_ns = (long long)c.timeout_ms * 1000000ll;
    P.idle_ns = (long long)c.idle_ms * 1000000ll;

    P.splits = 1;
    if (b1) {  // ---- batch-1 kernel: static schedule and packed weights
    if (nblk * KIE_TOPK_MAX > KIE_SAMPLE_VALS) {
        eng->fail(KIE_ERR_ARG, "the batch-1 kernel's sampling supports at most %d SMs", KIE_SAMPLE_VALS / KIE_TOPK_MAX);
        return bail(KIE_ERR_ARG);
    }
    if (d > KIE_B1_DMAX) {
        eng->fail(KIE_ERR_ARG, "the batch-1 kernel supports d_model <= %d", KIE_B1_DMAX);
        return bail(KIE_ERR_ARG);
    }
    // attention splits: about one (kv head, split) unit per CTA
    P.splits = std::max(1, nblk / Hkv);

    const int E = G * D;  // attention outputs of one kv head (its query heads)
    const bool f8 = c.weight_fp8 != 0;
    const int esz = f8 ? 1 : 2;
    P.wesz = esz;
    P.b1_tmem = b1_tm ? 1 : 0;
    P.b1_kvr = b1_kvr ? 1 : 0;
    const int Kph[KIE_NPH] = {d, 8, d, 8, d};
    std::vector<int> row0((size_t)KIE_NPH * (nblk + 1));
    // two rotation pairs at a time: a CTA's pairs then come as (dims i, i + 1), i even, of one
    // head, which its epilogue writes as single 32- or 64-bit words
    partition(&row0[PH_QKV * (nblk + 1)], (qd + 2 * kvd) / 4, 4, nblk);
    // O fold: CTA c = g * splits + s holds 8-column groups [s (E/8) / splits, (s+1) (E/8) / splits)
    // of kv head g's outputs, i.e. global groups g (E/8) + that; the CTAs past Hkv * splits none
    for (int cc = 0; cc <= nblk; cc++) {
        const int u = std::min(cc, Hkv * P.splits), g = u / P.splits, sp = u % P.splits;
        row0[PH_OF * (nblk + 1) + cc] = g * (E / 8) + (int)((long long)sp * (E / 8) / P.splits);
    }
    partition(&row0[PH_GU * (nblk + 1)], F / 8, 16, nblk);  // 8 gate/up pairs (16 rows) at a time
    partition(&row0[PH_DF * (nblk + 1)], F / 8, 1, nblk);   // the same pairs: 8-column groups of Wd
    partition(&row0[PH_HEAD * (nblk + 1)], V, 1, nblk);
    auto range = [&](int ph, int cc) { return row0[ph * (nblk + 1) + cc + 1] - row0[ph * (nblk + 1) + cc]; };
    for (int ph = 0; ph < KIE_NPH; ph++) {
        P.K[ph] = Kph[ph];
        const bool fold = (ph == PH_OF || ph == PH_DF);
        // rows per ring chunk (even for the paired phases), or 8-column groups per chunk of a fold
        P.cr[ph] = fold ? KIE_SLOT_BYTES / (d * 8 * esz) : kie_b1_chunk_rows(Kph[ph]) * (2 / esz);
        const int lim = fold ? KIE_FOLD_MAX / 8 : kie_b1_max_rows(Kph[ph]);
        for (int cc = 0; cc < nblk; cc++)
            if (range(ph, cc) > lim) {
                eng->fail(KIE_ERR_ARG, "phase %d gives a CTA more than %d %s", ph, lim, fold ? "column groups" : "rows");
                return bail(KIE_ERR_ARG);
            }
    }

    // ---- packed weights: CTA c's stream is one contiguous segment (per layer: QKV rows, its Wo
    // column groups, its gate/up rows, its Wd column groups; then its LM-head rows)
    std::vector<long long> seg_off(nblk + 1, 0);
    for (int cc = 0; cc < nblk; cc++) {
        const long long lb = ((long long)range(PH_QKV, cc) * d + (long long)range(PH_OF, cc) * d * 8 +
                              (long long)range(PH_GU, cc) * d + (long long)range(PH_DF, cc) * d * 8) * esz;
        seg_off[cc + 1] = seg_off[cc] + (long long)L * lb + (long long)range(PH_HEAD, cc) * d * esz;
    }
    uint8_t *wpack = nullptr;
    CKC(eng->alloc(&wpack, (size_t)seg_off[nblk]), "cudaMalloc packed weights");
    P.wpack = wpack;
    // E4M3 codes and row scales of every matrix (layer l, list index j; the LM head at [L][0]),
    // made once here and freed after the repack
    std::vector<uint8_t *> qcodes((size_t)(L + 1) * 9, nullptr);
    std::vector<float *> qscale((size_t)(L + 1) * 9, nullptr);
    auto free_q = [&]() {
        for (auto p : qcodes) cudaFree(p);
        for (auto p : qscale) cudaFree(p);
    };
    auto mat_shape = [&](int j, int *N, int *K) {
        switch (j) {
            case 1: *N = qd; *K = d; break;
            case 2: case 3: *N = kvd; *K = d; break;
            case 4: *N = d; *K = qd; break;
            case 6: case 7: *N = F; *K = d; break;
            default: *N = d; *K = F; break;  // 8: w_down
        }
    };
    if (f8) {
        for (int l = 0; l <= L && e == cudaSuccess; l++)
            for (int j = (l < L ? 1 : 0); j < (l < L ? 9 : 1) && e == cudaSuccess; j++) {
                if (j == 5) continue;  // the MLP norm gain
                int N = V, K = d;
                if (l < L) mat_shape(j, &N, &K);
                const void *src = l < L ? w->layers[(size_t)9 * l + j] : w->lm_head;
                e = cudaMalloc(&qcodes[(size_t)9 * l + j], (size_t)N * K);
                if (e == cudaSuccess) e = cudaMalloc(&qscale[(size_t)9 * l + j], (size_t)N * 4);
                if (e == cudaSuccess) e = kie_fp8_quantize(src, N, K, c.dtype, qcodes[(size_t)9 * l + j],
                                                           qscale[(size_t)9 * l + j], 0);
            }
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        if (e != cudaSuccess) {
            free_q();
            return bail(eng->cuda_fail(e, "weight quantisation"));
        }
        // the row scales in each phase's logical row order: per layer [QKV | O | gate/up | down],
        // then the LM head
        P.sc_stride = qd + 2 * kvd + d + 2 * F + d;
        std::vector<float> sc((size_t)L * P.sc_stride + V);
        std::vector<std::vector<float>> hs((size_t)(L + 1) * 9);
        for (int l = 0; l <= L && e == cudaSuccess; l++)
            for (int j = (l < L ? 1 : 0); j < (l < L ? 9 : 1) && e == cudaSuccess; j++) {
                if (j == 5) continue;
                int N = V, K = d;
                if (l < L) mat_shape(j, &N, &K);
                hs[(size_t)9 * l + j].resize(N);
                e = cudaMemcpy(hs[(size_t)9 * l + j].data(), qscale[(size_t)9 * l + j], (size_t)N * 4, cudaMemcpyDeviceToHost);
            }
        if (e != cudaSuccess) {
            free_q();
            return bail(eng->cuda_fail(e, "reading the row scales"));
        }
        for (int l = 0; l < L; l++) {
            float *o = sc.data() + (size_t)l * P.sc_stride;
            for (int r = 0; r < qd + 2 * kvd; r++) {
                int m, row;
                qkv_row(c, r, &m, &row);
                o[r] = hs[(size_t)9 * l + m][row];
            }
            o += qd + 2 * kvd;
            for (int r = 0; r < d; r++) o[r] = hs[(size_t)9 * l + 4][r];
            o += d;
            for (int r = 0; r < 2 * F; r++) o[r] = hs[(size_t)9 * l + ((r & 1) ? 7 : 6)][r >> 1];
            o += 2 * F;
            for (int r = 0; r < d; r++) o[r] = hs[(size_t)9 * l + 8][r];
        }
        for (int r = 0; r < V; r++) sc[(size_t)L * P.sc_stride + r] = hs[(size_t)9 * L][r];
        float *d_sc = nullptr;
        e = eng->alloc(&d_sc, sc.size() * 4);
        if (e == cudaSuccess) e = cudaMemcpy(d_sc, sc.data(), sc.size() * 4, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) {
            free_q();
            return bail(eng->cuda_fail(e, "row scales"));
        }
        P.wsc = d_sc;
    }
    // a matrix's rows as the repack reads them: the 16-bit weights, or their codes
    auto mat_src = [&](int l, int j) -> const uint8_t * {
        if (f8) return qcodes[(size_t)9 * l + j];
        return static_cast<const uint8_t *>(l < L ? w->layers[(size_t)9 * l + j] : w->lm_head);
    };
    {
        std::vector<RowCopy> rc;   // whole rows (GEMV phases)
        std::vector<FoldCopy> fc;  // column-group blocks (folds)
        rc.reserve((size_t)L * (qd + 2 * kvd + 2 * F) + V);
        for (int cc = 0; cc < nblk; cc++) {
            long long off = seg_off[cc];
            for (int l = 0; l <= L; l++) {
                for (int ph = (l < L ? 0 : PH_HEAD); ph < (l < L ? PH_HEAD : KIE_NPH); ph++) {
                    const int a = row0[ph * (nblk + 1) + cc], n = range(ph, cc);
                    if (ph == PH_OF || ph == PH_DF) {
                        if (n > 0) {
                            const uint8_t *src = mat_src(l, ph == PH_OF ? 4 : 8);
                            fc.push_back({off, src, (long long)(ph == PH_OF ? qd : F) * esz, 8 * a, n, d, esz});
                        }
                        off += (long long)n * d * 8 * esz;
                        continue;
                    }
                    const int K = Kph[ph];
                    for (int r = a; r < a + n; r++) {
                        const uint8_t *src;
                        if (ph == PH_QKV) {
                            int m, row;
                            qkv_row(c, r, &m, &row);
                            src = mat_src(l, m) + (size_t)row * K * esz;
                        } else if (ph == PH_GU) {
                            src = mat_src(l, (r & 1) ? 7 : 6) + (size_t)(r >> 1) * K * esz;
                        } else {
                            src = mat_src(L, 0) + (size_t)r * K * esz;
                        }
                        rc.push_back({off, src, (long long)K * esz});
                        off += (long long)K * esz;
                    }
                }
            }
            if (off != seg_off[cc + 1]) {
                free_q();
                eng->fail(KIE_ERR_ARG, "internal: segment size mismatch");
                return bail(KIE_ERR_ARG);
            }
        }
        RowCopy *d_rc = nullptr;
        FoldCopy *d_fc = nullptr;
        e = cudaMalloc(&d_rc, rc.size() * sizeof(RowCopy));
        if (e == cudaSuccess) e = cudaMalloc(&d_fc, std::max<size_t>(1, fc.size()) * sizeof(FoldCopy));
        if (e == cudaSuccess) e = cudaMemcpy(d_rc, rc.data(), rc.size() * sizeof(RowCopy), cudaMemcpyHostToDevice);
        if (e == cudaSuccess && !fc.empty())
            e = cudaMemcpy(d_fc, fc.data(), fc.size() * sizeof(FoldCopy), cudaMemcpyHostToDevice);
        if (e == cudaSuccess) {
            gather_rows_kernel<<<4 * nblk, 256>>>(d_rc, (long long)rc.size(), wpack);
            if (!fc.empty()) fold_pack_kernel<<<4 * nblk, 256>>>(d_fc, (long long)fc.size(), wpack);
            e = cudaGetLastError();
        }
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        cudaFree(d_rc);
        cudaFree(d_fc);
        free_q();
        if (e != cudaSuccess) return bail(eng->cuda_fail(e, "weight repack"));
    }
    int *d_row0 = nullptr;
    long long *d_seg = nullptr;
    CKC(eng->alloc(&d_row0, row0.size() * sizeof(int)), "cudaMalloc plan");
    CKC(eng->alloc(&d_seg, seg_off.size() * sizeof(long long)), "cudaMalloc plan");
    CKC(cudaMemcpy(d_row0, row0.data(), row0.size() * sizeof(int), cudaMemcpyHostToDevice), "upload plan");
    CKC(cudaMemcpy(d_seg, seg_off.data(), seg_off.size() * sizeof(long long), cudaMemcpyHostToDevice), "upload plan");
    P.row0 = d_row0;
    P.seg_off = d_seg;
    }  // batch-1 kernel

    if (mr) {  // ---- tick kernel: swizzled 128 x 64 tiles, tile ranges per SM and phase
        const int NGm = 5;
        const int Nm[NGm] = {qd + 2 * kvd, d, 2 * F, d, V};
        const int Km[NGm] = {d, qd, d, F, d};
        // work unit ("atom"): the tiles of two consecutive 64-wide k-steps of a 128-row block (the
        // odd last k-step of a block alone), moved by one bulk copy; atoms are split evenly over
        // the SMs, phase by phase
        auto natk = [&](int g) { return (Km[g] / 64 + 1) / 2; };
        auto atom_tiles = [&](int g, long long a) { return std::min(2, Km[g] / 64 - 2 * (int)(a % natk(g))); };
        std::vector<int> a0((size_t)NGm * (nblk + 1));
        for (int g = 0; g < NGm; g++) {
            const long long atoms = (long long)((Nm[g] + 127) / 128) * natk(g);
            for (int cc = 0; cc <= nblk; cc++) a0[(size_t)g * (nblk + 1) + cc] = (int)(cc * atoms / nblk);
        }
        std::vector<long long> mseg(nblk + 1, 0);
        for (int cc = 0; cc < nblk; cc++) {
            long long tiles = 0;
            for (int g = 0; g < NGm; g++) {
                long long n = 0;
                for (long long a = a0[(size_t)g * (nblk + 1) + cc]; a < a0[(size_t)g * (nblk + 1) + cc + 1]; a++)
                    n += atom_tiles(g, a);
                tiles += g < 4 ? n * L : n;
            }
            mseg[cc + 1] = mseg[cc] + tiles * 16384;
        }
        uint8_t *mpack = nullptr;
        CKC(eng->alloc(&mpack, (size_t)mseg[nblk]), "cudaMalloc tick weights");
        const size_t tsz = kie_mr_tile_src_bytes();
        std::vector<uint8_t> desc((size_t)(mseg[nblk] / 16384) * tsz);
        size_t nt = 0;
        for (int cc = 0; cc < nblk; cc++) {
            long long off = mseg[cc];
            for (int l = 0; l <= L; l++) {
                const void *const *Lw = w->layers + (size_t)9 * (l < L ? l : 0);
                for (int g = (l < L ? 0 : 4); g < (l < L ? 4 : 5); g++) {
                    const void *src3[3] = {nullptr, nullptr, nullptr};
                    int n0 = Nm[g], n1 = Nm[g];
                    switch (g) {
                        case 0: src3[0] = Lw[1]; src3[1] = Lw[2]; src3[2] = Lw[3]; n0 = qd; n1 = qd + kvd; break;
                        case 1: src3[0] = Lw[4]; break;
                        case 2: src3[0] = Lw[6]; src3[1] = Lw[7]; n0 = F; n1 = 2 * F; break;
                        case 3: src3[0] = Lw[8]; break;
                        default: src3[0] = w->lm_head; break;
                    }
                    for (int a = a0[(size_t)g * (nblk + 1) + cc]; a < a0[(size_t)g * (nblk + 1) + cc + 1]; a++)
                        for (int t = 0; t < atom_tiles(g, a); t++) {
                            kie_mr_tile_src(&desc[nt * tsz], src3, n0, n1, off, Nm[g], Km[g], a / natk(g),
                                            2 * (a % natk(g)) + t);
                            nt++;
                            off += 16384;
                        }
                }
            }
        }
        void *d_desc = nullptr;
        CKC(cudaMalloc(&d_desc, desc.size()), "cudaMalloc tick repack list");
        e = cudaMemcpy(d_desc, desc.data(), desc.size(), cudaMemcpyHostToDevice);
        if (e == cudaSuccess) e = kie_mr_repack(d_desc, (long long)nt, mpack, 0);
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        cudaFree(d_desc);
        if (e != cudaSuccess) return bail(eng->cuda_fail(e, "tick weight repack"));
        int *d_a0 = nullptr;
        long long *d_mseg = nullptr;
        CKC(eng->alloc(&d_a0, a0.size() * sizeof(int)), "cudaMalloc tick plan");
        CKC(eng->alloc(&d_mseg, mseg.size() * sizeof(long long)), "cudaMalloc tick plan");
        CKC(cudaMemcpy(d_a0, a0.data(), a0.size() * sizeof(int), cudaMemcpyHostToDevice), "upload tick plan");
        CKC(cudaMemcpy(d_mseg, mseg.data(), mseg.size() * sizeof(long long), cudaMemcpyHostToDevice), "upload tick plan");
        P.mr_wpack = mpack;
        P.mr_a0 = d_a0;
        P.mr_seg_off = d_mseg;
        const int R = 64;  // rows per step
        CKC(eng->alloc(&P.mr_x, (size_t)R * d * 4), "cudaMalloc tick scratch");
        CKC(eng->alloc(&P.mr_yqkv, (size_t)R * (qd + 2 * kvd) * 4), "cudaMalloc tick scratch");
        CKC(eng->alloc(&P.mr_ygu, (size_t)R * 2 * F * 4), "cudaMalloc tick scratch");
        CKC(eng->alloc(&P.mr_q, (size_t)R * qd * 4), "cudaMalloc tick scratch");
        const size_t bpack = (size_t)std::max(std::max(d, qd), F) / 64 * 16384;  // one 16 KB tile per k-step
        CKC(eng->alloc(&P.mr_bpack, bpack), "cudaMalloc tick scratch");
        CKC(cudaMemset(P.mr_bpack, 0, bpack), "memset");
        CKC(eng->alloc(&P.mr_logits, (size_t)R * V * 4), "cudaMalloc tick scratch");
        CKC(eng->alloc(&P.mr_part, (size_t)R * Hkv * G * (D + 2) * 4), "cudaMalloc tick scratch");
        CKC(eng->alloc(&P.mr_cnt, (size_t)R * Hkv * 4), "cudaMalloc tick scratch");
        CKC(eng->alloc(&P.mr_sid, (size_t)R * 4), "cudaMalloc tick scratch");
        CKC(eng->alloc(&P.mr_pos, (size_t)R * 4), "cudaMalloc tick scratch");
        CKC(eng->alloc(&P.mr_tok, (size_t)R * 4), "cudaMalloc tick scratch");
        CKC(cudaMemset(P.mr_cnt, 0, (size_t)R * Hkv * 4), "memset");
        CKC(cudaMemset(P.mr_x, 0, (size_t)R * d * 4), "memset");
    }

    // ---- small weights: embedding table and norm gains
    uint16_t *emb = nullptr, *gains = nullptr;
    CKC(eng->alloc(&emb, (size_t)V * d * 2), "cudaMalloc embedding");
    CKC(cudaMemcpy(emb, w->tok_emb, (size_t)V * d * 2, cudaMemcpyDeviceToDevice), "copy embedding");
    CKC(eng->alloc(&gains, (size_t)(2 * L + 1) * d * 2), "cudaMalloc gains");
    for (int l = 0; l < L; l++) {
        CKC(cudaMemcpy(gains + (size_t)(2 * l) * d, w->layers[9 * l + 0], (size_t)d * 2, cudaMemcpyDeviceToDevice), "gains");
        CKC(cudaMemcpy(gains + (size_t)(2 * l + 1) * d, w->layers[9 * l + 5], (size_t)d * 2, cudaMemcpyDeviceToDevice), "gains");
    }
    CKC(cudaMemcpy(gains + (size_t)(2 * L) * d, w->final_norm, (size_t)d * 2, cudaMemcpyDeviceToDevice), "gains");
    P.emb = emb;
    P.gains = gains;

    // ---- rotary table, computed in double on the host
    {
        std::vector<float2> rope((size_t)c.max_ctx * (D / 2));
        for (int p = 0; p < c.max_ctx; p++)
            for (int i = 0; i < D / 2; i++) {
                const double ang = (double)p * std::pow((double)c.rope_theta, -2.0 * i / D);
                rope[(size_t)p * (D / 2) + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
            }
        float2 *d_rope = nullptr;
        CKC(eng->alloc(&d_rope, rope.size() * sizeof(float2)), "cudaMalloc rope");
        CKC(cudaMemcpy(d_rope, rope.data(), rope.size() * sizeof(float2), cudaMemcpyHostToDevice), "upload rope");
        P.rope = d_rope;
    }

    // ---- KV cache for every session slot
    P.sess_stride = (long long)L * Hkv * c.max_ctx * D;
    CKC(eng->alloc(&P.kcache, (size_t)c.max_sessions * P.sess_stride * 2), "cudaMalloc K cache");
    CKC(eng->alloc(&P.vcache, (size_t)c.max_sessions * P.sess_stride * 2), "cudaMalloc V cache");
    // the tick kernel's attention reads K and V tiles by 2-D TMA: each arena as [rows][D], rows
    // = sessions * L * Hkv * max_ctx (one per cached position), boxes of 128 rows x 64 dims,
    // 128-byte swizzled (the MMA operand layouts); head_dim not a multiple of 64 keeps the
    // CUDA-core attention. A tile's rows may run up to 127 past the last row (zero fill), so
    // every coordinate stays below 2^31.
    P.mr_kmap = P.mr_vmap = nullptr;
    const unsigned long long kv_rows = (unsigned long long)c.max_sessions * L * Hkv * c.max_ctx;
    if (mr && D % 64 == 0 && kv_rows + 256 < (1ull << 31)) {
        // the driver's encoder, looked up through the runtime (no link-time driver dependency)
        typedef CUresult (*EncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                        const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                        CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        CKC(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q), "driver entry point");
        if (!fn || q != cudaDriverEntryPointSuccess) {
            eng->fail(KIE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
            return bail(KIE_ERR_CUDA);
        }
        CUtensorMap tm[2];
        const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)kv_rows};
        const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
        const cuuint32_t box[2] = {64, 128}, estr[2] = {1, 1};
        for (int a = 0; a < 2; a++) {
            const CUresult r = reinterpret_cast<EncodeTiled>(fn)(
                &tm[a], c.dtype == KIE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                a == 0 ? P.kcache : P.vcache, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            if (r != CUDA_SUCCESS) {
                eng->fail(KIE_ERR_CUDA, "cuTensorMapEncodeTiled (%s arena) failed: %d", a == 0 ? "K" : "V", (int)r);
                return bail(KIE_ERR_CUDA);
            }
        }
        uint8_t *d_map = nullptr;
        CKC(eng->alloc(&d_map, 2 * sizeof(CUtensorMap)), "cudaMalloc tensor maps");
        CKC(cudaMemcpy(d_map, tm, 2 * sizeof(CUtensorMap), cudaMemcpyHostToDevice), "upload tensor maps");
        P.mr_kmap = d_map;
        P.mr_vmap = d_map + sizeof(CUtensorMap);
    }

    // ---- activations and scratch
    CKC(eng->alloc(&P.x, (size_t)d * 4), "cudaMalloc x");
    CKC(eng->alloc(&P.q, (size_t)qd * 4), "cudaMalloc q");
    CKC(eng->alloc(&P.part, (size_t)Hkv * P.splits * G * (D + 2) * 4), "cudaMalloc partials");
    CKC(eng->alloc(&P.cnt, (size_t)Hkv * 4), "cudaMalloc counters");
    CKC(eng->alloc(&P.cand_val, (size_t)nblk * 4), "cudaMalloc candidates");
    CKC(eng->alloc(&P.cand_idx, (size_t)nblk * 4), "cudaMalloc candidates");
    CKC(eng->alloc(&P.cand_tv, (size_t)nblk * KIE_TOPK_MAX * 4), "cudaMalloc sampling candidates");
    CKC(eng->alloc(&P.cand_ti, (size_t)nblk * KIE_TOPK_MAX * 4), "cudaMalloc sampling candidates");
    {
        SampleCfg *samp = nullptr;
        CKC(eng->alloc(&samp, (size_t)c.max_sessions * sizeof(SampleCfg)), "cudaMalloc sampling settings");
        std::vector<SampleCfg> greedy(c.max_sessions, SampleCfg{1.f, 1, 0ull});
        CKC(cudaMemcpy(samp, greedy.data(), greedy.size() * sizeof(SampleCfg), cudaMemcpyHostToDevice), "sampling settings");
        P.samp = samp;
    }
    CKC(eng->alloc(&P.tokbuf, (size_t)c.max_ctx * 4), "cudaMalloc token buffer");
    CKC(eng->alloc(&P.bar, 32), "cudaMalloc barrier");  // [0]: grid barrier, [2]: the residual-read split barrier
    P.rd = P.bar + 2;
    CKC(eng->alloc(&P.err, 16), "cudaMalloc error word");
    CKC(eng->alloc(&P.last_seq, 16), "cudaMalloc sequence");
    CKC(eng->alloc(&P.cmd, sizeof(KieCmd)), "cudaMalloc command");
    CKC(cudaMemset(P.cnt, 0, (size_t)Hkv * 4), "memset");
    CKC(cudaMemset(P.bar, 0, 32), "memset");
    CKC(cudaMemset(P.err, 0, 16), "memset");
    CKC(cudaMemset(P.last_seq, 0, 16), "memset");
    CKC(cudaMemset(P.x, 0, (size_t)d * 4), "memset");

    // ---- the doorbell: mapped, pinned host memory
    eng->io_ints = 2 * (int64_t)c.max_ctx + 3 * 64 + 64 * 64;
    const size_t mb_bytes = sizeof(KieMailbox) + (size_t)eng->io_ints * 4;
    CKC(cudaHostAlloc((void **)&eng->mbox_host, mb_bytes, cudaHostAllocMapped | cudaHostAllocPortable), "cudaHostAlloc mailbox");
    memset(eng->mbox_host, 0, mb_bytes);
    CKC(cudaHostGetDevicePointer((void **)&eng->mbox_dev, eng->mbox_host, 0), "mailbox device alias");
    P.mbox = eng->mbox_dev;

    CKC(cudaStreamCreateWithFlags(&eng->stream, cudaStreamNonBlocking), "cudaStreamCreate");
    CKC(cudaEventCreateWithFlags(&eng->ev_done, cudaEventDisableTiming), "cudaEventCreate");
    CKC(cudaDeviceSynchronize(), "create");
    eng->sess_len.assign(c.max_sessions, 0);
    eng->sess_used.assign(c.max_sessions, 0);
    *out = eng;
    return KIE_OK;
}
#undef CKC

// ---------------------------------------------------------------- resident kernel control

static bool kernel_running(kie_engine *eng) {
    if (eng->resident == KIND_NONE) return false;
    const cudaError_t q = cudaEventQuery(eng->ev_done);
    if (q == cudaErrorNotReady) return true;
    eng->resident = KIND_NONE;
    return false;
}

static kie_status check_device_error(kie_engine *eng) {
    unsigned err = 0;
    cudaError_t e = cudaMemcpy(&err, eng->P.err, 4, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return eng->fail(KIE_ERR_DEVICE, "reading device status: %s", cudaGetErrorString(e));
#ifdef KIE_CHECK_BOUNDS
    if (!err) {
        const int bad = eng->check_guards();
        if (bad >= 0) return eng->fail(KIE_ERR_DEVICE, "guard words of engine buffer %d overwritten", bad);
    }
#endif
    if (err) {
        const unsigned code = err >> 8, where = err & 0xFF;
        const char *what = code == DERR_BARRIER_TIMEOUT ? "grid barrier timed out"
                           : code == DERR_RING_TIMEOUT  ? "weight ring wait timed out"
                           : code == DERR_BAD_TOKEN     ? "token id out of range"
                           : code == DERR_MMA_TIMEOUT   ? "tensor-core wait timed out"
                           : code == DERR_BOUNDS        ? "write index out of range (diagnostic build)"
                                                        : "unknown device error";
        return eng->fail(code == DERR_BARRIER_TIMEOUT || code == DERR_RING_TIMEOUT || code == DERR_MMA_TIMEOUT
                             ? KIE_ERR_TIMEOUT
                             : KIE_ERR_DEVICE,
                         "device: %s (phase %u)", what, where);
    }
    return KIE_OK;
}

static kie_status launch_resident(kie_engine *eng, int kind) {
    cudaError_t e = eng->reset_barrier(eng->stream);
    if (e == cudaSuccess) {
        KieCmd none{};
        e = kind == KIND_MR ? kie_mr_launch(eng->P, none, 1, eng->stream) : kie_b1_launch(eng->P, none, 1, eng->stream);
    }
    if (e == cudaSuccess) e = cudaEventRecord(eng->ev_done, eng->stream);
    if (e != cudaSuccess) return eng->cuda_fail(e, "launching the resident kernel");
    eng->resident = kind;
    return KIE_OK;
}

// Posts one command and waits for its completion (relaunching the kernel if it had gone idle).
static kie_status doorbell(kie_engine *eng, const KieCmd &cmd_in, int kind) {
    if (kernel_running(eng) && eng->resident != kind) {
        // another kernel is resident: ask it to leave first (handled by the caller's kind switch)
    }
    if (!kernel_running(eng)) {
        kie_status s = launch_resident(eng, kind);
        if (s != KIE_OK) return s;
    }
    KieMailbox *mb = eng->mbox_host;
    const uint32_t s = ++eng->seq;
    KieCmd cmd = cmd_in;
    cmd.seq = s;
    memcpy((void *)&mb->cmd, &cmd, sizeof cmd);
    std::atomic_thread_fence(std::memory_order_release);
    mb->cmd_seq = s;
    // the device's first wait of a command (the broadcast barrier) is bounded by idle + timeout
    const double t0 = now_s(), limit = (eng->cfg.timeout_ms + eng->cfg.idle_ms) * 1e-3;
    unsigned spins = 0;
    for (;;) {
        if (mb->done_seq == s) break;
        if ((++spins & 1023u) == 0) {
            if (!kernel_running(eng)) {
                std::atomic_thread_fence(std::memory_order_acquire);
                if (mb->done_seq == s) break;
                const kie_status ds = check_device_error(eng);
                if (ds != KIE_OK) return ds;
                const cudaError_t le = cudaGetLastError();
                if (le != cudaSuccess) return eng->fail(KIE_ERR_DEVICE, "resident kernel: %s", cudaGetErrorString(le));
                if (cmd.op == OP_EXIT) break;
                kie_status ls = launch_resident(eng, kind);  // it went idle before taking the command
                if (ls != KIE_OK) return ls;
            }
            // the time limit scales with the work of the command, with room for the device to
            // report its own timeout first
            const double budget = 1.5 * limit * (1.0 + (cmd.n > 0 ? cmd.n / 64.0 : 0.0));
            if (now_s() - t0 > budget) {
                return eng->fail(KIE_ERR_TIMEOUT, "no answer from the device after %.1f s", now_s() - t0);
            }
        } else {
            _mm_pause();
        }
    }
    std::atomic_thread_fence(std::memory_order_acquire);
    if (mb->status != 0) {
        const kie_status ds = check_device_error(eng);
        return ds != KIE_OK ? ds : eng->fail(KIE_ERR_DEVICE, "device reported a failed command");
    }
    return KIE_OK;
}

static kie_status stop_resident(kie_engine *eng) {
    if (!kernel_running(eng)) return KIE_OK;
    KieCmd ex{};
    ex.op = OP_EXIT;
    kie_status s = doorbell(eng, ex, eng->resident);
    const double t0 = now_s();
    while (kernel_running(eng)) {
        if (now_s() - t0 > eng->cfg.timeout_ms * 1e-3) return eng->fail(KIE_ERR_TIMEOUT, "resident kernel did not stop");
    }
    return s;
}

extern "C" void kie_destroy(kie_engine *eng) {
    if (!eng) return;
    if (!eng->poisoned && eng->stream) stop_resident(eng);
    if (eng->stream) cudaStreamSynchronize(eng->stream);
    for (void *p : eng->dev_allocs) cudaFree(p);
    if (eng->P.trace) cudaFree(eng->P.trace);
    if (eng->mbox_host) cudaFreeHost(eng->mbox_host);
    if (eng->ev_done) cudaEventDestroy(eng->ev_done);
    if (eng->stream) cudaStreamDestroy(eng->stream);
    delete eng;
}

// ---------------------------------------------------------------- sessions

static kie_status check_live(kie_engine *eng) {
    if (!eng) return KIE_ERR_ARG;
    if (eng->poisoned) return KIE_ERR_STATE;
    return KIE_OK;
}

static kie_status check_sid(kie_engine *eng, int32_t sid) {
    if (sid < 0 || sid >= eng->cfg.max_sessions || !eng->sess_used[sid])
        return eng->fail(KIE_ERR_ARG, "session %d is not open", sid);
    return KIE_OK;
}

static kie_status set_sampling(kie_engine *eng, int32_t sid, const SampleCfg &sc);

extern "C" kie_status kie_session_open(kie_engine *eng, int32_t *sid) {
    kie_status s = check_live(eng);
    if (s != KIE_OK) return s;
    if (!sid) return KIE_ERR_ARG;
    for (int i = 0; i < eng->cfg.max_sessions; i++)
        if (!eng->sess_used[i]) {
            if ((s = set_sampling(eng, i, SampleCfg{1.f, 1, 0ull})) != KIE_OK) return s;  // greedy
            eng->sess_used[i] = 1;
            eng->sess_len[i] = 0;
            *sid = i;
            return KIE_OK;
        }
    return eng->fail(KIE_ERR_CAPACITY, "all %d session slots are open", eng->cfg.max_sessions);
}

static kie_status set_sampling(kie_engine *eng, int32_t sid, const SampleCfg &sc) {
    // the legacy default stream: it does not wait for the engine's (non-blocking) stream, where
    // a resident kernel may sit idle between commands
    const cudaError_t e = cudaMemcpy(const_cast<SampleCfg *>(eng->P.samp) + sid, &sc, sizeof sc, cudaMemcpyHostToDevice);
    return e == cudaSuccess ? KIE_OK : eng->cuda_fail(e, "sampling settings");
}

extern "C" kie_status kie_session_sampling(kie_engine *eng, int32_t sid, const kie_sampling *sp) {
    kie_status s = check_live(eng);
    if (s != KIE_OK) return s;
    if ((s = check_sid(eng, sid)) != KIE_OK) return s;
    SampleCfg sc{1.f, 1, 0ull};
    if (sp) {
        if (sp->top_k < 1 || sp->top_k > std::min(KIE_TOPK_MAX, eng->cfg.vocab))
            return eng->fail(KIE_ERR_ARG, "top_k must be in [1, %d]", std::min(KIE_TOPK_MAX, eng->cfg.vocab));
        if (sp->top_k > 1) {
            if (!(sp->temperature > 0.f) || !std::isfinite(sp->temperature) || !std::isfinite(1.f / sp->temperature))
                return eng->fail(KIE_ERR_ARG, "temperature must be a positive finite number");
            sc = SampleCfg{1.f / sp->temperature, sp->top_k, (unsigned long long)sp->seed};
        }
    }
    return set_sampling(eng, sid, sc);
}

extern "C" kie_status kie_session_close(kie_engine *eng, int32_t sid) {
    kie_status s = check_live(eng);
    if (s != KIE_OK) return s;
    if ((s = check_sid(eng, sid)) != KIE_OK) return s;
    eng->sess_used[sid] = 0;
    eng->sess_len[sid] = 0;
    return KIE_OK;
}

extern "C" kie_status kie_session_length(kie_engine *eng, int32_t sid, int32_t *ctx) {
    if (!eng || !ctx) return KIE_ERR_ARG;
    kie_status s = check_sid(eng, sid);
    if (s != KIE_OK) return s;
    *ctx = eng->sess_len[sid];
    return KIE_OK;
}

extern "C" kie_status kie_session_rewind(kie_engine *eng, int32_t sid, int32_t ctx) {
    kie_status s = check_live(eng);
    if (s != KIE_OK) return s;
    if ((s = check_sid(eng, sid)) != KIE_OK) return s;
    if (ctx < 0 || ctx > eng->sess_len[sid]) return eng->fail(KIE_ERR_ARG, "rewind past the current length");
    eng->sess_len[sid] = ctx;
    return KIE_OK;
}

extern "C" kie_status kie_session_kv(kie_engine *eng, int32_t sid, void **k_dev, void **v_dev) {
    if (!eng || !k_dev || !v_dev) return KIE_ERR_ARG;
    kie_status s = check_sid(eng, sid);
    if (s != KIE_OK) return s;
    *k_dev = eng->P.kcache + (size_t)sid * eng->P.sess_stride;
    *v_dev = eng->P.vcache + (size_t)sid * eng->P.sess_stride;
    return KIE_OK;
}

// ---------------------------------------------------------------- decode calls

static kie_status ensure_kind(kie_engine *eng, int kind) {
    if (kernel_running(eng) && eng->resident != kind) return stop_resident(eng);
    return KIE_OK;
}

static kie_status check_tokens(kie_engine *eng, const int32_t *t, int n) {
    for (int i = 0; i < n; i++)
        if (t[i] < 0 || t[i] >= eng->cfg.vocab) return eng->fail(KIE_ERR_ARG, "token %d out of range", t[i]);
    return KIE_OK;
}

static int32_t *io_dev(kie_engine *eng, int64_t at) { return eng->mbox_dev->io + at; }

extern "C" kie_status kie_prefill(kie_engine *eng, int32_t sid, const int32_t *tokens, int32_t n, int32_t *first_token) {
    kie_status s = check_live(eng);
    if (s != KIE_OK) return s;
    if (!tokens || !first_token || n <= 0) return eng->fail(KIE_ERR_ARG, "prefill needs n >= 1 tokens");
    if ((s = check_sid(eng, sid)) != KIE_OK) return s;
    if ((s = check_tokens(eng, tokens, n)) != KIE_OK) return s;
    const int ctx = eng->sess_len[sid];
    if ((int64_t)ctx + n > eng->cfg.max_ctx) return eng->fail(KIE_ERR_CAPACITY, "prefill of %d at %d exceeds max_ctx", n, ctx);
    if (eng->cfg.modes & KIE_MODE_TICK) {
        // chunks of up to 64 consecutive positions run as rows of the tick kernel
        if ((s = ensure_kind(eng, KIND_MR)) != KIE_OK) return s;
        for (int c0 = 0; c0 < n; c0 += 64) {
            const int m = std::min(64, n - c0);
            int32_t *io = eng->mbox_host->io;
            for (int j = 0; j < m; j++) {
                io[j] = sid;
                io[64 + j] = ctx + c0 + j;
                io[128 + j] = tokens[c0 + j];
            }
            KieCmd cmd{};
            cmd.op = OP_PREFILL;
            cmd.sid = sid;
            cmd.n = 1;
            cmd.n_sess = m;
            cmd.flags = (c0 + m == n) ? 1 : 0;  // logits only after the last chunk
            cmd.tokens = io_dev(eng, 0);
            cmd.out = io_dev(eng, 192);
            s = doorbell(eng, cmd, KIND_MR);
            if (s != KIE_OK) return s;
            eng->sess_len[sid] = ctx + c0 + m;
        }
        *first_token = ((volatile int32_t *)eng->mbox_host->io)[192];
        return KIE_OK;
    }
    if ((s = ensure_kind(eng, KIND_B1)) != KIE_OK) return s;
    memcpy(eng->mbox_host->io, tokens, (size_t)n * 4);
    KieCmd cmd{};
    cmd.op = OP_PREFILL;
    cmd.sid = sid;
    cmd.pos0 = ctx;
    cmd.n = n;
    cmd.tokens = io_dev(eng, 0);
    cmd.out = io_dev(eng, eng->cfg.max_ctx);
    s = doorbell(eng, cmd, KIND_B1);
    if (s != KIE_OK) return s;
    *first_token = ((volatile int32_t *)eng->mbox_host->io)[eng->cfg.max_ctx];
    eng->sess_len[sid] = ctx + n;
    return KIE_OK;
}

static kie_status decode_doorbell(kie_engine *eng, int32_t sid, int32_t in_token, int32_t n, int32_t *out,
                                  float *logits_dev) {
    kie_status s = check_live(eng);
    if (s != KIE_OK) return s;
    if (!out || n <= 0) return eng->fail(KIE_ERR_ARG, "need n >= 1 and an output buffer");
    if ((s = check_sid(eng, sid)) != KIE_OK) return s;
    if ((s = check_tokens(eng, &in_token, 1)) != KIE_OK) return s;
    const int ctx = eng->sess_len[sid];
    if ((int64_t)ctx + n > eng->cfg.max_ctx) return eng->fail(KIE_ERR_CAPACITY, "%d steps at %d exceed max_ctx", n, ctx);
    if ((int64_t)n > eng->io_ints - eng->cfg.max_ctx) return eng->fail(KIE_ERR_ARG, "n too large for the mailbox");
    if (!(eng->cfg.modes & KIE_MODE_BATCH1)) return eng->fail(KIE_ERR_UNSUPPORTED, "engine built without KIE_MODE_BATCH1");
    if ((s = ensure_kind(eng, KIND_B1)) != KIE_OK) return s;
    KieCmd cmd{};
    cmd.op = OP_DECODE;
    cmd.sid = sid;
    cmd.pos0 = ctx;
    cmd.n = n;
    cmd.in_tok = in_token;
    cmd.out = io_dev(eng, eng->cfg.max_ctx);
    cmd.logits = logits_dev;
    s = doorbell(eng, cmd, KIND_B1);
    if (s != KIE_OK) return s;
    const volatile int32_t *io = eng->mbox_host->io + eng->cfg.max_ctx;
    for (int i = 0; i < n; i++) out[i] = io[i];
    eng->sess_len[sid] = ctx + n;
    return KIE_OK;
}

extern "C" kie_status kie_decode_step(kie_engine *eng, int32_t sid, int32_t in_token, int32_t *out_token,
                                      float *logits_dev) {
    return decode_doorbell(eng, sid, in_token, 1, out_token, logits_dev);
}

extern "C" kie_status kie_generate(kie_engine *eng, int32_t sid, int32_t in_token, int32_t n, int32_t *out_tokens) {
    return decode_doorbell(eng, sid, in_token, n, out_tokens, nullptr);
}

extern "C" kie_status kie_decode_launch(kie_engine *eng, int32_t sid, const int32_t *in_token_dev, int32_t n,
                                        int32_t *out_tokens_dev, float *logits_dev, void *stream) {
    kie_status s = check_live(eng);
    if (s != KIE_OK) return s;
    if (!in_token_dev || !out_tokens_dev || n <= 0) return eng->fail(KIE_ERR_ARG, "launch needs device buffers and n >= 1");
    if ((s = check_sid(eng, sid)) != KIE_OK) return s;
    const int ctx = eng->sess_len[sid];
    if ((int64_t)ctx + n > eng->cfg.max_ctx) return eng->fail(KIE_ERR_CAPACITY, "%d steps at %d exceed max_ctx", n, ctx);
    if (!(eng->cfg.modes & KIE_MODE_BATCH1)) return eng->fail(KIE_ERR_UNSUPPORTED, "engine built without KIE_MODE_BATCH1");
    if ((s = stop_resident(eng)) != KIE_OK) return s;
    cudaStream_t st = stream ? static_cast<cudaStream_t>(stream) : eng->stream;
    KieCmd cmd{};
    cmd.op = OP_DECODE;
    cmd.sid = sid;
    cmd.pos0 = ctx;
    cmd.n = n;
    cmd.tok_dev = in_token_dev;
    cmd.out = out_tokens_dev;
    cmd.logits = logits_dev;
    cudaError_t e = eng->reset_barrier(st);
    if (e == cudaSuccess) e = kie_b1_launch(eng->P, cmd, 0, st);
    if (e != cudaSuccess) return eng->cuda_fail(e, "launching the decode kernel");
    eng->sess_len[sid] = ctx + n;
    return KIE_OK;
}

extern "C" kie_status kie_sync(kie_engine *eng) {
    kie_status s = check_live(eng);
    if (s != KIE_OK) return s;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return eng->fail(KIE_ERR_DEVICE, "kernel failed: %s", cudaGetErrorString(e));
    return check_device_error(eng);
}

// Checks shared by the two tick entry points.
static kie_status tick_checks(kie_engine *eng, int32_t n_sess, const int32_t *sids, int32_t steps) {
    if (!(eng->cfg.modes & KIE_MODE_TICK)) return eng->fail(KIE_ERR_UNSUPPORTED, "engine built without KIE_MODE_TICK");
    if (n_sess < 1 || n_sess > 64 || steps < 1 || steps > 64 || !sids)
        return eng->fail(KIE_ERR_ARG, "tick needs 1..64 sessions and 1..64 steps");
    std::vector<char> seen(eng->cfg.max_sessions, 0);
    kie_status s;
    for (int i = 0; i < n_sess; i++) {
        if ((s = check_sid(eng, sids[i])) != KIE_OK) return s;
        if (seen[sids[i]]) return eng->fail(KIE_ERR_ARG, "session %d appears twice in one tick", sids[i]);
        seen[sids[i]] = 1;
        if ((int64_t)eng->sess_len[sids[i]] + steps > eng->cfg.max_ctx)
            return eng->fail(KIE_ERR_CAPACITY, "session %d: %d steps exceed max_ctx", sids[i], steps);
    }
    return KIE_OK;
}

extern "C" kie_status kie_tick_launch(kie_engine *eng, int32_t n_sess, const int32_t *sids, const int32_t *in_tokens_dev,
                                      int32_t steps, int32_t *out_tokens_dev, float *logits_dev, void *stream) {
    kie_status s = check_live(eng);
    if (s != KIE_OK) return s;
    if (!in_tokens_dev || !out_tokens_dev) return eng->fail(KIE_ERR_ARG, "tick launch needs device buffers");
    if ((s = tick_checks(eng, n_sess, sids, steps)) != KIE_OK) return s;
    if ((s = stop_resident(eng)) != KIE_OK) return s;
    cudaStream_t st = stream ? static_cast<cudaStream_t>(stream) : eng->stream;
    // rows of the command: sessions and positions from the host (pageable: copied before return)
    std::vector<int32_t> sp(2 * n_sess);
    for (int i = 0; i < n_sess; i++) {
        sp[i] = sids[i];
        sp[n_sess + i] = eng->sess_len[sids[i]];
    }
    cudaError_t e = cudaMemcpyAsync(eng->P.mr_sid, sp.data(), (size_t)n_sess * 4, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(eng->P.mr_pos, sp.data() + n_sess, (size_t)n_sess * 4, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(eng->P.mr_tok, in_tokens_dev, (size_t)n_sess * 4, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = eng->reset_barrier(st);
    KieCmd cmd{};
    cmd.op = OP_TICK;
    cmd.n = steps;
    cmd.n_sess = n_sess;
    cmd.out = out_tokens_dev;
    cmd.logits = logits_dev;
    if (e == cudaSuccess) e = kie_mr_launch(eng->P, cmd, 0, st);
    if (e != cudaSuccess) return eng->cuda_fail(e, "launching the tick kernel");
    for (int i = 0; i < n_sess; i++) eng->sess_len[sids[i]] += steps;
    return KIE_OK;
}

extern "C" kie_status kie_tick(kie_engine *eng, int32_t n_sess, const int32_t *sids, const int32_t *in_tokens,
                               int32_t steps, int32_t *out_tokens, float *logits_dev) {
    kie_status s = check_live(eng);
    if (s != KIE_OK) return s;
    if (!in_tokens || !out_tokens) return eng->fail(KIE_ERR_ARG, "tick needs host buffers");
    if ((s = tick_checks(eng, n_sess, sids, steps)) != KIE_OK) return s;
    if ((s = check_tokens(eng, in_tokens, n_sess)) != KIE_OK) return s;
    if ((s = ensure_kind(eng, KIND_MR)) != KIE_OK) return s;
    int32_t *io = eng->mbox_host->io;
    for (int i = 0; i < n_sess; i++) {
        io[i] = sids[i];
        io[64 + i] = eng->sess_len[sids[i]];
        io[128 + i] = in_tokens[i];
    }
    KieCmd cmd{};
    cmd.op = OP_TICK;
    cmd.n = steps;
    cmd.n_sess = n_sess;
    cmd.tokens = io_dev(eng, 0);
    cmd.out = io_dev(eng, 192);
    cmd.logits = logits_dev;
    s = doorbell(eng, cmd, KIND_MR);
    if (s != KIE_OK) return s;
    const volatile int32_t *out = eng->mbox_host->io + 192;
    for (int i = 0; i < steps * n_sess; i++) out_tokens[i] = out[i];
    for (int i = 0; i < n_sess; i++) eng->sess_len[sids[i]] += steps;
    return KIE_OK;
}

// ---------------------------------------------------------------- fault injection (tests)

extern "C" kie_status kie_inject_fault(kie_engine *eng, int32_t fault) {
    kie_status s = check_live(eng);
    if (s != KIE_OK) return s;
    if (fault != KIE_FAULT_NONE && fault != KIE_FAULT_BARRIER_SHORT) return eng->fail(KIE_ERR_ARG, "unknown fault %d", fault);
    if ((s = stop_resident(eng)) != KIE_OK) return s;  // the fault applies to a fresh launch
    eng->pending_fault = fault;
    return KIE_OK;
}

// ---------------------------------------------------------------- phase trace

extern "C" int32_t kie_trace_events(kie_engine *eng) {
    if (!eng) return 0;
    return 1 + 16 * eng->cfg.n_layers + 3 + KIE_NPH + 1;
}

extern "C" kie_status kie_trace_enable(kie_engine *eng, int32_t tokens) {
    kie_status s = check_live(eng);
    if (s != KIE_OK) return s;
    if (tokens < 0 || tokens > 4096) return eng->fail(KIE_ERR_ARG, "trace tokens must be in [0, 4096]");
    if ((s = stop_resident(eng)) != KIE_OK) return s;
    cudaDeviceSynchronize();
    if (eng->P.trace) {
        cudaFree(eng->P.trace);
        eng->P.trace = nullptr;
    }
    eng->P.trace_tokens = tokens;
    eng->P.trace_events = kie_trace_events(eng);
    if (tokens > 0) {
        const size_t n = (size_t)eng->nblk * tokens * eng->P.trace_events;
        cudaError_t e = cudaMalloc(&eng->P.trace, n * 8);
        if (e == cudaSuccess) e = cudaMemset(eng->P.trace, 0, n * 8);
        if (e != cudaSuccess) {
            eng->P.trace = nullptr;
            eng->P.trace_tokens = 0;
            return eng->cuda_fail(e, "trace buffer");
        }
    }
    return KIE_OK;
}

extern "C" kie_status kie_trace_read(kie_engine *eng, uint64_t *host, int64_t max_elems, int64_t *n) {
    kie_status s = check_live(eng);
    if (s != KIE_OK) return s;
    if (!n || (!host && max_elems > 0)) return KIE_ERR_ARG;
    const int64_t total = eng->P.trace ? (int64_t)eng->nblk * eng->P.trace_tokens * eng->P.trace_events : 0;
    *n = total;
    if (!total || max_elems <= 0) return KIE_OK;
    if ((s = stop_resident(eng)) != KIE_OK) return s;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemcpy(host, eng->P.trace, (size_t)std::min(total, max_elems) * 8, cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? KIE_OK : eng->cuda_fail(e, "reading the trace");
}
