// SIMT kernels of the fp32 workload: the fp32 GEMM, epilogue passes over an
// fp32 GEMM result, and a CUDA-core causal flash attention.
//
// The fp32 workload is compared at 1e-4 RMS, which rules out TF32 tensor
// cores; its GEMMs run as plain fp32 FMA tiles.
#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

// C[M, N] (+)= A[M, K] . W[N, K]^T, 64x64 tile, 256 threads, 4x4 per thread.
template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const T* __restrict__ A, const T* __restrict__ W,
                                                        float* __restrict__ C, int M, int N, int K,
                                                        int accumulate) {
    __shared__ float As[16][68];
    __shared__ float Ws[16][68];
    const int bm = blockIdx.y * 64, bn = blockIdx.x * 64;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 16) {
        for (int i = tid; i < 64 * 16; i += 256) {
            const int r = i >> 4, kk = i & 15;
            As[kk][r] = (bm + r < M && k0 + kk < K) ? to_f32(A[(size_t)(bm + r) * K + k0 + kk]) : 0.f;
            Ws[kk][r] = (bn + r < N && k0 + kk < K) ? to_f32(W[(size_t)(bn + r) * K + k0 + kk]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = Ws[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = bm + ty * 4 + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = bn + tx * 4 + j;
            if (n >= N) continue;
            float* p = C + (size_t)m * N + n;
            *p = accumulate ? *p + acc[i][j] : acc[i][j];
        }
    }
}

int launch_gemm_simt(int dtype, const void* A, const void* W, float* C, int M, int N, int K, int accumulate,
                     cudaStream_t st) {
    if (M <= 0 || N <= 0) return LLAMA_OK;
    dim3 grid(ceil_div(N, 64), ceil_div(M, 64));
    if (dtype == LLAMA_BF16)
        gemm_simt_kernel<bf16><<<grid, 256, 0, st>>>((const bf16*)A, (const bf16*)W, C, M, N, K, accumulate);
    else
        gemm_simt_kernel<float><<<grid, 256, 0, st>>>((const float*)A, (const float*)W, C, M, N, K, accumulate);
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}

// Epilogue pass over an fp32 GEMM result C [M, ldc]: one thread per
// (row, 32-column chunk).
template <typename T, int MODE>
__global__ void epilogue_from_f32_kernel(const float* __restrict__ C, int ldc, EpiArgs a) {
    const int chunks = (MODE == EPI_SWIGLU ? a.hidden : a.N) / 32;
    const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (idx >= (int64_t)a.M * chunks) return;
    const int m = (int)(idx / chunks);
    const int c = (int)(idx - (int64_t)m * chunks);
    const float* row = C + (size_t)m * ldc;
    if (MODE == EPI_SWIGLU) {
        const int j0 = c * 32;
        const int ng = (j0 / 128) * 256 + (j0 % 128);
        float g[32], u[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            g[j] = row[ng + j];
            u[j] = row[ng + 128 + j];
        }
        epi_swiglu32<T>(a, m, j0, g, u);
    } else {
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = row[c * 32 + j];
        if constexpr (MODE == EPI_RESID) epi_resid32(a, m, c * 32, v);
        else epi_qkv32<T>(a, m, c * 32, v);
    }
}

int launch_epilogue_from_f32(int dtype, int mode, const float* C, int ldc, const EpiArgs& a, cudaStream_t st) {
    const int chunks = (mode == EPI_SWIGLU ? a.hidden : a.N) / 32;
    const int64_t total = (int64_t)a.M * chunks;
    if (total == 0) return LLAMA_OK;
    const int blocks = (int)((total + 127) / 128);
    if (mode == EPI_SWIGLU) {
        if (dtype == LLAMA_BF16) epilogue_from_f32_kernel<bf16, EPI_SWIGLU><<<blocks, 128, 0, st>>>(C, ldc, a);
        else epilogue_from_f32_kernel<float, EPI_SWIGLU><<<blocks, 128, 0, st>>>(C, ldc, a);
    } else if (mode == EPI_QKV) {
        if (dtype == LLAMA_BF16) epilogue_from_f32_kernel<bf16, EPI_QKV><<<blocks, 128, 0, st>>>(C, ldc, a);
        else epilogue_from_f32_kernel<float, EPI_QKV><<<blocks, 128, 0, st>>>(C, ldc, a);
    } else if (mode == EPI_RESID) {
        epilogue_from_f32_kernel<float, EPI_RESID><<<blocks, 128, 0, st>>>(C, ldc, a);
    } else {
        return LLAMA_ERR_INVALID_ARG;
    }
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}

// ---------------------------------------------------------------------------
// CUDA-core causal flash attention (online softmax), one CTA per
// (64-query tile, head, sequence); key tiles above the diagonal are skipped.
// q: [B][H][S][HD]; k, v: [B][Hkv][kv_stride][HD] (query head h reads key/value
// head h / (H / Hkv)); o: [B*S][H*HD].
template <typename T, int HD>
__global__ void __launch_bounds__(256) attn_prefill_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                                const T* __restrict__ v, T* __restrict__ o,
                                                                int H, int Hkv, int S, int kv_stride,
                                                                float scale) {
    constexpr int BQ = 64, BK = 64, LD = HD + 1, CPT = HD / 16;
    extern __shared__ float sm[];
    float* Qs = sm;                 // [BQ][LD]
    float* Ks = Qs + BQ * LD;       // [BK][LD]
    float* Vs = Ks + BK * LD;       // [BK][LD]
    float* Ps = Vs + BK * LD;       // [BQ][BK+1]
    const int qt = (gridDim.x - 1) - blockIdx.x;   // longest tiles first
    const int h = blockIdx.y, b = blockIdx.z;
    const int q0 = qt * BQ;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const size_t head = (size_t)b * H + h;
    const size_t kv_head = (size_t)b * Hkv + h / (H / Hkv);
    const T* qh = q + head * S * HD;
    const T* kh = k + kv_head * (size_t)kv_stride * HD;
    const T* vh = v + kv_head * (size_t)kv_stride * HD;
    for (int i = tid; i < BQ * HD; i += 256) {
        const int r = i / HD, c = i % HD;
        Qs[r * LD + c] = (q0 + r < S) ? to_f32(qh[(size_t)(q0 + r) * HD + c]) * scale : 0.f;
    }
    float m_i[4], l_i[4], acc[4][CPT];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m_i[i] = -INFINITY;
        l_i[i] = 0.f;
#pragma unroll
        for (int j = 0; j < CPT; ++j) acc[i][j] = 0.f;
    }
    const int k_end = min(S, q0 + BQ);
    for (int k0 = 0; k0 < k_end; k0 += BK) {
        __syncthreads();
        for (int i = tid; i < BK * HD; i += 256) {
            const int r = i / HD, c = i % HD;
            const bool ok = k0 + r < S;
            Ks[r * LD + c] = ok ? to_f32(kh[(size_t)(k0 + r) * HD + c]) : 0.f;
            Vs[r * LD + c] = ok ? to_f32(vh[(size_t)(k0 + r) * HD + c]) : 0.f;
        }
        __syncthreads();
        float s[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) s[i][j] = 0.f;
        for (int c = 0; c < HD; ++c) {
            float a[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = Qs[(ty * 4 + i) * LD + c];
#pragma unroll
            for (int j = 0; j < 4; ++j) bb[j] = Ks[(tx * 4 + j) * LD + c];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) s[i][j] = fmaf(a[i], bb[j], s[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = q0 + ty * 4 + i;
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int jj = k0 + tx * 4 + j;
                if (jj > t || jj >= S) s[i][j] = -INFINITY;
                mx = fmaxf(mx, s[i][j]);
            }
#pragma unroll
            for (int off = 1; off < 16; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_new = fmaxf(m_i[i], mx);
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            const float corr = __expf(m_i[i] - m_use);
            float rs = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float p = __expf(s[i][j] - m_use);
                Ps[(ty * 4 + i) * (BK + 1) + tx * 4 + j] = p;
                rs += p;
            }
#pragma unroll
            for (int off = 1; off < 16; off <<= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
            l_i[i] = l_i[i] * corr + rs;
            m_i[i] = m_new;
#pragma unroll
            for (int j = 0; j < CPT; ++j) acc[i][j] *= corr;
        }
        __syncthreads();
        for (int kk = 0; kk < BK; ++kk) {
            float p[4], vv[CPT];
#pragma unroll
            for (int i = 0; i < 4; ++i) p[i] = Ps[(ty * 4 + i) * (BK + 1) + kk];
#pragma unroll
            for (int j = 0; j < CPT; ++j) vv[j] = Vs[kk * LD + tx * CPT + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < CPT; ++j) acc[i][j] = fmaf(p[i], vv[j], acc[i][j]);
        }
    }
    const int d = H * HD;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = q0 + ty * 4 + i;
        if (t >= S) continue;
        const float inv = 1.f / l_i[i];
        T* orow = o + ((size_t)b * S + t) * d + (size_t)h * HD + tx * CPT;
#pragma unroll
        for (int j = 0; j < CPT; ++j) orow[j] = from_f32<T>(acc[i][j] * inv);
    }
}

template <typename T, int HD>
static int attn_simt_attr(size_t smem) {
    static PerDeviceOnce once;
    return once_per_device(once, [smem]() -> int {
        LLAMA_CUDA_TRY(cudaFuncSetAttribute(attn_prefill_simt_kernel<T, HD>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        return (int)LLAMA_OK;
    });
}

template <typename T, int HD>
static size_t attn_simt_smem() {
    return (size_t)(3 * 64 * (HD + 1) + 64 * 65) * sizeof(float);
}

int attention_prepare() {
    int rc;
    if ((rc = attn_simt_attr<float, 128>(attn_simt_smem<float, 128>()))) return rc;
    if ((rc = attn_simt_attr<float, 64>(attn_simt_smem<float, 64>()))) return rc;
    return attn_simt_attr<float, 32>(attn_simt_smem<float, 32>());
}

template <typename T, int HD>
static int launch_attn_simt_t(const void* q, const void* k, const void* v, void* o, int B, int H, int Hkv,
                              int S, int kv_stride, cudaStream_t st) {
    const size_t smem = attn_simt_smem<T, HD>();
    int rc = attn_simt_attr<T, HD>(smem);
    if (rc) return rc;
    dim3 grid(ceil_div(S, 64), H, B);
    attn_prefill_simt_kernel<T, HD><<<grid, 256, smem, st>>>((const T*)q, (const T*)k, (const T*)v, (T*)o, H, Hkv,
                                                             S, kv_stride, 1.0f / sqrtf((float)HD));
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}

int launch_attention_prefill_simt(int dtype, const void* q, const void* k, const void* v, void* o, int B,
                                  int H, int Hkv, int S, int hd, int kv_stride, cudaStream_t st) {
    if (B <= 0 || S <= 0) return LLAMA_OK;
    if (Hkv <= 0 || H % Hkv != 0) return LLAMA_ERR_INVALID_ARG;
    if (dtype != LLAMA_F32) return LLAMA_ERR_INVALID_ARG;   // bf16 runs on the tensor cores (attn_tc.cu)
    if (hd == 128) return launch_attn_simt_t<float, 128>(q, k, v, o, B, H, Hkv, S, kv_stride, st);
    if (hd == 64) return launch_attn_simt_t<float, 64>(q, k, v, o, B, H, Hkv, S, kv_stride, st);
    if (hd == 32) return launch_attn_simt_t<float, 32>(q, k, v, o, B, H, Hkv, S, kv_stride, st);
    return LLAMA_ERR_INVALID_ARG;
}
