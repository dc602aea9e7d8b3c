// Standalone split-K decode attention (kie_flash_decode): the attention device code of the
// decode megakernel, launched on its own over a caller-provided KV cache.
#include <cuda_runtime.h>

#include "kie_attn.cuh"

namespace {

constexpr int FD_WARPS = 8;

template <int DT>
__global__ void __launch_bounds__(FD_WARPS * 32) flash_decode_kernel(AttnArgs A, int G) {
    __shared__ AttnSmem S;
    attn_all_units<DT, FD_WARPS>(A, S, G, blockIdx.x, gridDim.x);
}

// Splits per kv head: about 64 positions per split, at most 64 splits.
int fd_splits(int G, int n_ctx) {
    (void)G;
    int s = (n_ctx + 63) / 64;
    if (s > 64) s = 64;
    return s < 1 ? 1 : s;
}

bool fd_shape_ok(int Hq, int Hkv, int D, int n_ctx, int dtype) {
    if (Hq <= 0 || Hkv <= 0 || n_ctx <= 0 || Hq % Hkv != 0 || Hq / Hkv > KIE_GMAX) return false;
    if (D != 8 && D != 16 && D != 32 && D != 64 && D != 128) return false;
    return dtype == KIE_FP16 || dtype == KIE_BF16;
}

int64_t fd_part_bytes(int Hq, int Hkv, int D, int n_ctx) {
    const int G = Hq / Hkv;
    const int S = fd_splits(G, n_ctx);
    return ((int64_t)Hkv * S * G * (D + 2) * 4 + 255) / 256 * 256;
}

}  // namespace

extern "C" int64_t kie_flash_decode_scratch_bytes(int32_t n_heads, int32_t n_kv_heads, int32_t head_dim,
                                                  int32_t n_ctx) {
    if (!fd_shape_ok(n_heads, n_kv_heads, head_dim, n_ctx, KIE_FP16)) return -1;
    return fd_part_bytes(n_heads, n_kv_heads, head_dim, n_ctx) + (int64_t)n_kv_heads * 4;
}

extern "C" kie_status kie_flash_decode(const float *q_dev, const void *k_dev, const void *v_dev, int32_t n_heads,
                                       int32_t n_kv_heads, int32_t head_dim, int32_t n_ctx, int64_t kv_stride,
                                       int32_t dtype, float *out_dev, void *scratch_dev, int64_t scratch_bytes,
                                       void *stream) {
    if (!fd_shape_ok(n_heads, n_kv_heads, head_dim, n_ctx, dtype) || kv_stride < n_ctx) return KIE_ERR_ARG;
    if (!q_dev || !k_dev || !v_dev || !out_dev || !scratch_dev) return KIE_ERR_ARG;
    if (scratch_bytes < kie_flash_decode_scratch_bytes(n_heads, n_kv_heads, head_dim, n_ctx)) return KIE_ERR_ARG;
    const int G = n_heads / n_kv_heads;
    AttnArgs A;
    A.q = q_dev;
    A.k = static_cast<const uint16_t *>(k_dev);
    A.v = static_cast<const uint16_t *>(v_dev);
    A.head_stride = kv_stride * head_dim;
    A.part = static_cast<float *>(scratch_dev);
    A.cnt = reinterpret_cast<unsigned *>(static_cast<char *>(scratch_dev) +
                                         fd_part_bytes(n_heads, n_kv_heads, head_dim, n_ctx));
    A.o = out_dev;
    A.bpack = nullptr;
    A.brow = 0;
    A.gout = -1;
    A.cnt_target = 0;
    A.oslice = nullptr;  // the last split merges
    A.timeout_ns = 0;
    A.err = nullptr;
    A.D = head_dim;
    A.Hkv = n_kv_heads;
    A.nsplit = fd_splits(G, n_ctx);
    A.ctx = n_ctx;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(A.cnt, 0, (size_t)n_kv_heads * 4, s) != cudaSuccess) return KIE_ERR_CUDA;
    const dim3 grid(n_kv_heads * A.nsplit);
    if (dtype == KIE_BF16) flash_decode_kernel<KIE_BF16><<<grid, FD_WARPS * 32, 0, s>>>(A, G);
    else flash_decode_kernel<KIE_FP16><<<grid, FD_WARPS * 32, 0, s>>>(A, G);
    return cudaGetLastError() == cudaSuccess ? KIE_OK : KIE_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------
// Allocation-free variant of kie_flash_decode.
//
// Some callers must not allocate device memory while they run: code that works inside a
// memory budget fixed at start-up (no allocator after initialisation, as in a resident
// serving loop), code whose device memory belongs to another framework's allocator, and
// latency-critical loops where cudaMalloc/cudaFree would stall the device. They call this
// entry point instead: the split partials and merge counters live in one static device
// array of KIE_FLASH_DECODE_NOALLOC_MAX_BYTES that every GPU loading this library keeps
// until the process exits.
// ---------------------------------------------------------------------------------------

#include <mutex>

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KIE_FLASH_DECODE_NOALLOC_MAX_BYTES];

constexpr int NOALLOC_MAX_DEVICES = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[NOALLOC_MAX_DEVICES];  // device address of the array, per device (set up once)

// The host-side symbol is only a stand-in: the kernel needs the array's device address,
// looked up once per device with that device current.
cudaError_t noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" kie_status kie_flash_decode_noalloc(const float *q_dev, const void *k_dev, const void *v_dev,
                                               int32_t n_heads, int32_t n_kv_heads, int32_t head_dim, int32_t n_ctx,
                                               int64_t kv_stride, int32_t dtype, float *out_dev, void *stream) {
    if (!fd_shape_ok(n_heads, n_kv_heads, head_dim, n_ctx, dtype) || kv_stride < n_ctx) return KIE_ERR_ARG;
    if (!q_dev || !k_dev || !v_dev || !out_dev) return KIE_ERR_ARG;
    const int64_t need = kie_flash_decode_scratch_bytes(n_heads, n_kv_heads, head_dim, n_ctx);
    if (need > (int64_t)KIE_FLASH_DECODE_NOALLOC_MAX_BYTES) return KIE_ERR_CAPACITY;
    void *scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) return KIE_ERR_CUDA;
    // the same launch as kie_flash_decode, with the static array as its scratch
    return kie_flash_decode(q_dev, k_dev, v_dev, n_heads, n_kv_heads, head_dim, n_ctx, kv_stride, dtype, out_dev,
                            scratch, (int64_t)KIE_FLASH_DECODE_NOALLOC_MAX_BYTES, stream);
}
