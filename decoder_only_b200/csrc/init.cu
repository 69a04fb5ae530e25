// Device-side random initialisation of the weights.
//
// The same published generator the synthetic workloads are defined with,
// implemented here independently for the device:
//   Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): ten rounds of
//     (hi0,lo0) = mulhilo(0xD2511F53, x0); (hi1,lo1) = mulhilo(0xCD9E8D57, x2);
//     x = (hi1 ^ x1 ^ k0, lo1, hi0 ^ x3 ^ k1, lo0), key += (0x9E3779B9, 0xBB67AE85)
//     between rounds; key = (seed, tensor id).
//   Box-Muller (1958): element e uses counter (e >> 2, 0, 0, 0); lane e & 3
//     takes the pair p = (e & 3) >> 1 of the output words, u1 = (a+1) 2^-32,
//     u2 = b 2^-32, z = sqrt(-2 ln u1) * (cos | sin)(2 pi u2) for even | odd
//     lanes; the weight is 0.02 z in fp64, rounded to nearest-even into the
//     storage type directly from fp64.
// Element e is the row-major index of the matrix in the (d_in, d_out)
// orientation in which the forward pass computes x @ W (the embedding
// table: (vocab, d) row-major); the device stores the matrix K-major.
#include "common.cuh"
#include "kernels.h"

__device__ __forceinline__ void philox4x32_10(uint32_t x[4], uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint32_t hi0 = __umulhi(0xD2511F53u, x[0]), lo0 = 0xD2511F53u * x[0];
        uint32_t hi1 = __umulhi(0xCD9E8D57u, x[2]), lo1 = 0xCD9E8D57u * x[2];
        uint32_t y0 = hi1 ^ x[1] ^ k0;
        uint32_t y2 = hi0 ^ x[3] ^ k1;
        x[0] = y0;
        x[1] = lo1;
        x[2] = y2;
        x[3] = lo0;
    }
}

__device__ __forceinline__ double normal_at(uint32_t seed, uint32_t tensor_id, uint64_t e) {
    uint32_t x[4] = {(uint32_t)(e >> 2), (uint32_t)(e >> 34), 0u, 0u};
    philox4x32_10(x, seed, tensor_id);
    const int j = (int)(e & 3u);
    const uint32_t a = (j >> 1) ? x[2] : x[0];
    const uint32_t b = (j >> 1) ? x[3] : x[1];
    const double u1 = ((double)a + 1.0) * 2.3283064365386963e-10;
    const double u2 = (double)b * 2.3283064365386963e-10;
    const double R = sqrt(-2.0 * log(u1));
    const double t = 2.0 * 3.141592653589793 * u2;
    return (j & 1) ? R * sin(t) : R * cos(t);
}

// fp64 -> bf16, nearest-even, without double rounding: truncate to fp32,
// mark inexactness in the lowest bit (round to odd), then round fp32 -> bf16.
__device__ __forceinline__ bf16 f64_to_bf16_rne(double v) {
    float f = __double2float_rz(v);
    if ((double)f != v) f = __uint_as_float(__float_as_uint(f) | 1u);
    return __float2bfloat16_rn(f);
}

template <typename T> __device__ __forceinline__ T round_store(double v);
template <> __device__ __forceinline__ float round_store<float>(double v) { return __double2float_rn(v); }
template <> __device__ __forceinline__ bf16 round_store<bf16>(double v) { return f64_to_bf16_rne(v); }

// Fill the device rows of a block of one logical matrix.
//   The logical matrix has output columns n in [0, N_full) and inputs
//   k in [0, K_full); element index e = rowmajor_nk ? n*K_full + k
//   : k*N_full + n.  The block held here is n in [n0, n0 + N_loc),
//   k in [k0, k0 + K_loc) (a tensor-parallel shard; the whole matrix when
//   n0 = k0 = 0 and the sizes are the full ones).  Local column nl = n - n0
//   goes to device row row_off + (nl / blk) * blk_stride + (nl % blk), row
//   length K_loc, at column k - k0.
template <typename T>
__global__ void init_matrix_kernel(T* __restrict__ dst, int K_full, int N_full, int k0, int K_loc, int n0, int N_loc,
                                   int blk, int blk_stride, int row_off, int rowmajor_nk, uint32_t seed,
                                   uint32_t tensor_id, double scale) {
    const uint64_t total = (uint64_t)N_loc * (uint64_t)K_loc;
    for (uint64_t idx = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (uint64_t)gridDim.x * blockDim.x) {
        const int nl = (int)(idx / (uint64_t)K_loc);
        const int kl = (int)(idx - (uint64_t)nl * K_loc);
        const uint64_t n = (uint64_t)(n0 + nl), k = (uint64_t)(k0 + kl);
        const uint64_t e = rowmajor_nk ? n * K_full + k : k * N_full + n;
        const int row = row_off + (nl / blk) * blk_stride + (nl % blk);
        dst[(size_t)row * K_loc + kl] = round_store<T>(scale * normal_at(seed, tensor_id, e));
    }
}

__global__ void fill_f32_kernel(float* dst, float v, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = v;
}

int launch_init_shard(int dtype, void* dst, int K_full, int N_full, int k0, int K_loc, int n0, int N_loc, int blk,
                      int blk_stride, int row_off, int rowmajor_nk, uint32_t seed, uint32_t tensor_id, double scale,
                      cudaStream_t st) {
    if (k0 < 0 || n0 < 0 || K_loc <= 0 || N_loc <= 0 || k0 + K_loc > K_full || n0 + N_loc > N_full || blk <= 0)
        return LLAMA_ERR_INVALID_ARG;
    const int threads = 256;
    const int blocks = 148 * 16;
    if (dtype == LLAMA_BF16)
        init_matrix_kernel<bf16><<<blocks, threads, 0, st>>>((bf16*)dst, K_full, N_full, k0, K_loc, n0, N_loc, blk,
                                                             blk_stride, row_off, rowmajor_nk, seed, tensor_id, scale);
    else
        init_matrix_kernel<float><<<blocks, threads, 0, st>>>((float*)dst, K_full, N_full, k0, K_loc, n0, N_loc,
                                                              blk, blk_stride, row_off, rowmajor_nk, seed, tensor_id,
                                                              scale);
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}

int launch_init_matrix(int dtype, void* dst, int K, int N_log, int blk, int blk_stride, int row_off,
                       int rowmajor_nk, uint32_t seed, uint32_t tensor_id, double scale,
                       cudaStream_t st) {
    return launch_init_shard(dtype, dst, K, N_log, 0, K, 0, N_log, blk, blk_stride, row_off, rowmajor_nk, seed,
                             tensor_id, scale, st);
}

int launch_fill_f32(float* dst, float v, int64_t n, cudaStream_t st) {
    fill_f32_kernel<<<148 * 4, 256, 0, st>>>(dst, v, n);
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}

// c[r] = b[r] + sum_k W[r][k] beta[k] (fp32 accumulate), one warp per row:
// the folded bias of a projection that consumes a shifted RMSNorm.
template <typename T>
__global__ void bias_fold_kernel(const T* __restrict__ W, int rows, int K, const float* __restrict__ beta,
                                 const float* __restrict__ b, float* __restrict__ c) {
    const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (r >= rows) return;
    const T* w = W + (size_t)r * K;
    float s = 0.f;
    for (int k = lane; k < K; k += 32) s = fmaf(to_f32(w[k]), beta[k], s);
    s = warp_sum(s);
    if (lane == 0) c[r] = b[r] + s;
}

int launch_bias_fold(int dtype, const void* W, int rows, int K, const float* beta, const float* b, float* c,
                     cudaStream_t st) {
    const int blocks = (rows + 7) / 8;
    if (dtype == LLAMA_BF16)
        bias_fold_kernel<bf16><<<blocks, 256, 0, st>>>((const bf16*)W, rows, K, beta, b, c);
    else
        bias_fold_kernel<float><<<blocks, 256, 0, st>>>((const float*)W, rows, K, beta, b, c);
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}
