// FP8 (E4M3) weights for the batch-1 kernel: per-row quantisation of a 16-bit matrix.
//
// Quantisation halves the bytes a decode step streams ("The path to ubiquitous AI (17k
// tokens/sec)", best practice 2: advanced model quantisation). Each row n of W [rows][cols]
// gets the scale s_n = max_k |W[n][k]| / 448 (fp32; 1 for an all-zero row) and the codes
// q[n][k] = E4M3(W[n][k] / s_n), the fp32 quotient rounded to the nearest code (ties to even)
// and saturated at +-448, the largest finite E4M3 value. A matrix-vector product then uses
// value(q[n][k]) * s_n.
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "kie_device.cuh"

namespace {

constexpr int QT = 256;

template <int DT>
__global__ void __launch_bounds__(QT) quantize_rows_kernel(const uint16_t *w, long long rows, int cols, uint8_t *q,
                                                           float *scale) {
    __shared__ float red[QT / 32];
    for (long long n = blockIdx.x; n < rows; n += gridDim.x) {
        const uint16_t *row = w + n * cols;
        float amax = 0.f;
        for (int k = threadIdx.x; k < cols; k += QT) amax = fmaxf(amax, fabsf(cvt1<DT>(row[k])));
        amax = warp_max(amax);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
        __syncthreads();
        float m = 0.f;
        for (int i = 0; i < QT / 32; i++) m = fmaxf(m, red[i]);
        const float s = m > 0.f ? __fdiv_rn(m, 448.0f) : 1.0f;
        uint8_t *qr = q + n * cols;
        for (int k = threadIdx.x; k < cols; k += QT)
            qr[k] = (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(cvt1<DT>(row[k]), s), __NV_SATFINITE, __NV_E4M3);
        if (threadIdx.x == 0) scale[n] = s;
        __syncthreads();  // red is reused by the next row
    }
}

}  // namespace

extern "C++" cudaError_t kie_fp8_quantize(const void *w, long long rows, int cols, int dtype, uint8_t *q, float *scale,
                                          cudaStream_t stream) {
    if (rows <= 0) return cudaSuccess;
    const int grid = (int)(rows < 4096 ? rows : 4096);
    if (dtype == KIE_BF16)
        quantize_rows_kernel<KIE_BF16><<<grid, QT, 0, stream>>>(static_cast<const uint16_t *>(w), rows, cols, q, scale);
    else
        quantize_rows_kernel<KIE_FP16><<<grid, QT, 0, stream>>>(static_cast<const uint16_t *>(w), rows, cols, q, scale);
    return cudaGetLastError();
}

extern "C" kie_status kie_quantize_e4m3(const void *w_dev, int64_t rows, int32_t cols, int32_t dtype, uint8_t *q_dev,
                                        float *scale_dev, void *stream) {
    if (!w_dev || !q_dev || !scale_dev || rows < 0 || cols <= 0) return KIE_ERR_ARG;
    if (dtype != KIE_FP16 && dtype != KIE_BF16) return KIE_ERR_ARG;
    return kie_fp8_quantize(w_dev, rows, cols, dtype, q_dev, scale_dev, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? KIE_OK
               : KIE_ERR_CUDA;
}
