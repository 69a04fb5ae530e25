// Row kernels: embedding gather, RMSNorm + cast, greedy argmax.
//
// RMSNorm ("RMSNorm: LayerNorm minus the mean"; gain g from "An Architecture
// Recipe Without an Invention Myth"): y = x / sqrt(mean(x^2) + eps) * g,
// fp32 in, fp32 sum of squares, written in the GEMM operand type.  One CTA
// per row, 16-byte loads, the row kept in registers between the two passes,
// warp-shuffle + shared-memory reduction.  HBM-bound: 4d bytes read +
// (2 or 4)d bytes written per row.
#include "common.cuh"
#include "kernels.h"

template <typename T>
__global__ void embed_kernel(const int32_t* __restrict__ tok, const T* __restrict__ E, float* __restrict__ x,
                             int d, int vocab, int* __restrict__ err) {
    pdl_launch_dependents();
    pdl_wait();
    const int r = blockIdx.x;
    int t = tok[r];
    if (t < 0 || t >= vocab) {   // out-of-range id: flag it, read row 0 instead
        if (threadIdx.x == 0) atomicOr(err, 2);
        t = 0;
    }
    const T* e = E + (size_t)t * d;
    float* o = x + (size_t)r * d;
    for (int i = threadIdx.x; i < d; i += blockDim.x) o[i] = to_f32(e[i]);
}

template <typename TO>
__device__ __forceinline__ void store4(TO* p, float a, float b, float c, float d);
template <>
__device__ __forceinline__ void store4<float>(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
template <>
__device__ __forceinline__ void store4<bf16>(bf16* p, float a, float b, float c, float d) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(a, b), pack_bf16x2(c, d));
}

constexpr int RMS_MAXV = 8;   // float4 per thread held in registers: d <= 8 * 4 * 256 = 8192

template <typename TO>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const float* __restrict__ x, const float* __restrict__ g,
                                                      const float* __restrict__ beta, TO* __restrict__ y, int d,
                                                      float eps) {
    pdl_launch_dependents();
    pdl_wait();
    const int r = blockIdx.x;
    const int nv = d >> 2;
    const float4* xr = reinterpret_cast<const float4*>(x + (size_t)r * d);
    float4 v[RMS_MAXV];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < RMS_MAXV; ++j) {
        const int i = threadIdx.x + j * blockDim.x;
        if (i < nv) {
            v[j] = xr[i];
            ss += v[j].x * v[j].x + v[j].y * v[j].y + v[j].z * v[j].z + v[j].w * v[j].w;
        }
    }
    __shared__ float red[32];
    ss = warp_sum(ss);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) red[w] = ss;
    __syncthreads();
    if (w == 0) {
        float t = (l < (int)(blockDim.x >> 5)) ? red[l] : 0.f;
        t = warp_sum(t);
        if (l == 0) red[0] = t;
    }
    __syncthreads();
    const float inv = rsqrtf(red[0] / (float)d + eps);
    const float4* g4 = reinterpret_cast<const float4*>(g);
    TO* yr = y + (size_t)r * d;
#pragma unroll
    for (int j = 0; j < RMS_MAXV; ++j) {
        const int i = threadIdx.x + j * blockDim.x;
        if (i < nv) {
            const float4 gg = g4[i];
            const float4 bb = beta ? reinterpret_cast<const float4*>(beta)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
            store4<TO>(yr + 4 * i, v[j].x * inv * gg.x + bb.x, v[j].y * inv * gg.y + bb.y,
                       v[j].z * inv * gg.z + bb.z, v[j].w * inv * gg.w + bb.w);
        }
    }
}

int launch_rmsnorm(int dtype, const float* x, const float* g, void* y, int rows, int d, float eps,
                   cudaStream_t st, const float* beta) {
    if (rows <= 0) return LLAMA_OK;
    const int nv = d / 4;
    int threads = ((ceil_div(nv, 4) + 31) / 32) * 32;
    if (threads < 32) threads = 32;
    if (threads > 256) threads = 256;
    if (nv > RMS_MAXV * threads) return LLAMA_ERR_INVALID_ARG;
    if (dtype == LLAMA_BF16)
        launch_pdl(rmsnorm_kernel<bf16>, dim3(rows), dim3(threads), 0, st, x, g, beta, (bf16*)y, d, eps);
    else
        launch_pdl(rmsnorm_kernel<float>, dim3(rows), dim3(threads), 0, st, x, g, beta, (float*)y, d, eps);
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}

int launch_embed(int dtype, const int32_t* tok, const void* E, float* x, int rows, int d, int vocab, int* err,
                 cudaStream_t st) {
    if (rows <= 0) return LLAMA_OK;
    if (dtype == LLAMA_BF16)
        launch_pdl(embed_kernel<bf16>, dim3(rows), dim3(256), 0, st, tok, (const bf16*)E, x, d, vocab, err);
    else
        launch_pdl(embed_kernel<float>, dim3(rows), dim3(256), 0, st, tok, (const float*)E, x, d, vocab, err);
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}

// Greedy choice: argmax over a logits row, lowest index on ties.  One CTA per row.
__global__ void __launch_bounds__(256) argmax_kernel(const float* __restrict__ logits, int n, int64_t ld,
                                                     int32_t* __restrict__ out) {
    const int r = blockIdx.x;
    const float* p = logits + (size_t)r * ld;
    float best = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const float v = p[i];
        if (v > best || (v == best && i < bi) || (bi == 0x7fffffff && v != v)) {
            best = v;
            bi = i;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > best || (ov == best && oi < bi)) {
            best = ov;
            bi = oi;
        }
    }
    __shared__ float sb[8];
    __shared__ int si[8];
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) {
        sb[w] = best;
        si[w] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int k = 1; k < (int)(blockDim.x >> 5); ++k)
            if (sb[k] > best || (sb[k] == best && si[k] < bi)) {
                best = sb[k];
                bi = si[k];
            }
        out[r] = (bi == 0x7fffffff) ? 0 : bi;
    }
}

int launch_argmax(const float* logits, int rows, int n, int64_t ld, int32_t* out, cudaStream_t st) {
    if (rows <= 0) return LLAMA_OK;
    argmax_kernel<<<rows, 256, 0, st>>>(logits, n, ld, out);
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}

// Greedy choice over long rows: the row is cut into chunks of AMX_CHUNK
// logits, one CTA each; every CTA leaves its (max, lowest index) in the
// workspace and bumps the row's counter; the CTA that arrives last merges
// the chunks in index order (so ties still go to the lowest id) and resets
// the counter for the next launch.
constexpr int AMX_CHUNK = 2048;

__device__ __forceinline__ bool amx_better(float v, int i, float bv, int bi) {
    return v > bv || (v == bv && i < bi);
}

__global__ void __launch_bounds__(256) argmax_split_kernel(const float* __restrict__ logits, int n, int64_t ld,
                                                           int32_t* __restrict__ out, int2* __restrict__ part,
                                                           int* __restrict__ counters, int chunks) {
    pdl_launch_dependents();
    pdl_wait();
    const int r = blockIdx.y, c = blockIdx.x;
    const float* p = logits + (size_t)r * ld;
    const int i0 = c * AMX_CHUNK, i1 = min(n, i0 + AMX_CHUNK);
    float best = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
        const float v = p[i];
        if (amx_better(v, i, best, bi)) {
            best = v;
            bi = i;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (amx_better(ov, oi, best, bi)) {
            best = ov;
            bi = oi;
        }
    }
    __shared__ float sb[8];
    __shared__ int si[8];
    __shared__ int last;
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) {
        sb[w] = best;
        si[w] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int k = 1; k < (int)(blockDim.x >> 5); ++k)
            if (amx_better(sb[k], si[k], best, bi)) {
                best = sb[k];
                bi = si[k];
            }
        part[(size_t)r * chunks + c] = make_int2(__float_as_int(best), bi);
        __threadfence();
        const int prev = atomicAdd(counters + r, 1);
        last = (prev == chunks - 1);
        if (last) {
            counters[r] = 0;
            __threadfence();
            float fb = -INFINITY;
            int fi = 0x7fffffff;
            for (int k = 0; k < chunks; ++k) {
                const int2 e = __ldcg(part + (size_t)r * chunks + k);
                if (amx_better(__int_as_float(e.x), e.y, fb, fi)) {
                    fb = __int_as_float(e.x);
                    fi = e.y;
                }
            }
            out[r] = (fi == 0x7fffffff) ? 0 : fi;
        }
    }
}

int argmax_split_chunks(int n) { return (n + AMX_CHUNK - 1) / AMX_CHUNK; }

int launch_argmax_split(const float* logits, int rows, int n, int64_t ld, int32_t* out, int2* part, int* counters,
                        cudaStream_t st) {
    if (rows <= 0) return LLAMA_OK;
    const int chunks = argmax_split_chunks(n);
    launch_pdl(argmax_split_kernel, dim3(chunks, rows), dim3(256), 0, st, logits, n, ld, out, part, counters, chunks);
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}
