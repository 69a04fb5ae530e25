// Decode-side attention: split-sequence attention over the contiguous KV
// cache.
//
// Decode attention ("GQA Was Not an Original LLaMA Feature": every step
// reads the keys and values of all previous tokens) is HBM-bound: each
// (sequence, head) streams len * head_dim * 2 elements once.  The sequence
// is cut into chunks of 256 keys so that B*H*chunks CTAs cover the SMs; each
// chunk leaves (max, sum, unnormalised output) in the workspace and a second
// pass merges the chunks (the online-softmax merge rule).
#include <mutex>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

constexpr int DEC_CHUNK = 256;   // keys per CTA
constexpr int DEC_WARPS = 4;

template <typename T> struct Vec16;                      // 16 bytes of T
template <> struct Vec16<bf16> { static constexpr int N = 8; };
template <> struct Vec16<float> { static constexpr int N = 4; };

template <typename T>
__device__ __forceinline__ void load16(const T* p, float* out);
template <>
__device__ __forceinline__ void load16<bf16>(const bf16* p, float* out) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(p));
    float2 f;
    f = unpack_bf16x2(w.x); out[0] = f.x; out[1] = f.y;
    f = unpack_bf16x2(w.y); out[2] = f.x; out[3] = f.y;
    f = unpack_bf16x2(w.z); out[4] = f.x; out[5] = f.y;
    f = unpack_bf16x2(w.w); out[6] = f.x; out[7] = f.y;
}
template <>
__device__ __forceinline__ void load16<float>(const float* p, float* out) {
    const float4 w = __ldg(reinterpret_cast<const float4*>(p));
    out[0] = w.x; out[1] = w.y; out[2] = w.z; out[3] = w.w;
}

// Eight lanes share one key: lane (g*8 + r) holds dims [r*DPL, (r+1)*DPL).
template <typename T, int HD>
__global__ void __launch_bounds__(DEC_WARPS * 32) attn_decode_partial_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, int H, int len_static,
    const int* __restrict__ d_len_minus1, int kv_stride, float scale, float* __restrict__ work, int n_chunks) {
    constexpr int DPL = HD / 8;                 // dims per lane
    constexpr int VPL = DPL / Vec16<T>::N;      // 16-byte loads per lane per row
    pdl_launch_dependents();
    pdl_wait();
    const int len = d_len_minus1 ? (*d_len_minus1 + 1) : len_static;
    const int chunk = blockIdx.x;
    const int bh = blockIdx.y;                  // b*H + h
    const int b = bh / H, h = bh - b * H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 3, r = lane & 7;
    const int k_begin = chunk * DEC_CHUNK;
    const int k_stop = min(len, k_begin + DEC_CHUNK);

    float qv[DPL];
    {
        const T* qp = q + ((size_t)b * H + h) * HD + r * DPL;
#pragma unroll
        for (int u = 0; u < VPL; ++u) load16<T>(qp + u * Vec16<T>::N, qv + u * Vec16<T>::N);
#pragma unroll
        for (int j = 0; j < DPL; ++j) qv[j] *= scale;
    }
    float m = -INFINITY, l = 0.f, o[DPL];
#pragma unroll
    for (int j = 0; j < DPL; ++j) o[j] = 0.f;

    const size_t head_off = ((size_t)b * H + h) * (size_t)kv_stride * HD;
    const T* kh = k + head_off + r * DPL;
    const T* vh = v + head_off + r * DPL;
    // Warp w walks keys [k_begin + 64 w, k_begin + 64 w + 64) eight at a time:
    // lane group g takes keys jb + g and jb + 4 + g, so each lane has four
    // 16-byte-per-row loads (two K rows, two V rows) in flight per round.
    // jb is warp-uniform, so every lane takes part in the shuffles.
    const int seg_end = min(k_stop, k_begin + (warp + 1) * (DEC_CHUNK / DEC_WARPS));
    for (int jb = k_begin + warp * (DEC_CHUNK / DEC_WARPS); jb < seg_end; jb += 8) {
        const int j0 = jb + g, j1 = jb + 4 + g;
        const bool ok0 = j0 < seg_end, ok1 = j1 < seg_end;
        float k0[DPL], k1[DPL], x0[DPL], x1[DPL];
#pragma unroll
        for (int u = 0; u < VPL; ++u) {
            if (ok0) {
                load16<T>(kh + (size_t)j0 * HD + u * Vec16<T>::N, k0 + u * Vec16<T>::N);
                load16<T>(vh + (size_t)j0 * HD + u * Vec16<T>::N, x0 + u * Vec16<T>::N);
            }
            if (ok1) {
                load16<T>(kh + (size_t)j1 * HD + u * Vec16<T>::N, k1 + u * Vec16<T>::N);
                load16<T>(vh + (size_t)j1 * HD + u * Vec16<T>::N, x1 + u * Vec16<T>::N);
            }
        }
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int e = 0; e < DPL; ++e) {
            s0 = fmaf(qv[e], ok0 ? k0[e] : 0.f, s0);
            s1 = fmaf(qv[e], ok1 ? k1[e] : 0.f, s1);
        }
#pragma unroll
        for (int o2 = 1; o2 < 8; o2 <<= 1) {
            s0 += __shfl_xor_sync(0xffffffffu, s0, o2);
            s1 += __shfl_xor_sync(0xffffffffu, s1, o2);
        }
        if (!ok0) s0 = -INFINITY;
        if (!ok1) s1 = -INFINITY;
        const float m_new = fmaxf(m, fmaxf(s0, s1));
        if (m_new != -INFINITY) {
            const float corr = __expf(m - m_new);
            const float p0 = __expf(s0 - m_new), p1 = __expf(s1 - m_new);
            l = l * corr + p0 + p1;
#pragma unroll
            for (int e = 0; e < DPL; ++e)
                o[e] = fmaf(o[e], corr, fmaf(p0, ok0 ? x0[e] : 0.f, p1 * (ok1 ? x1[e] : 0.f)));
            m = m_new;
        }
    }
    // merge the 16 key groups (4 per warp x 4 warps) through shared memory
    __shared__ float sm_m[DEC_WARPS * 4], sm_l[DEC_WARPS * 4];
    __shared__ float sm_o[DEC_WARPS * 4][HD];
    const int grp = warp * 4 + g;
    if (r == 0) {
        sm_m[grp] = m;
        sm_l[grp] = l;
    }
#pragma unroll
    for (int e = 0; e < DPL; ++e) sm_o[grp][r * DPL + e] = o[e];
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int t = 0; t < DEC_WARPS * 4; ++t) M = fmaxf(M, sm_m[t]);
    float* wp = work + ((size_t)bh * n_chunks + chunk) * (HD + 2);
    for (int c = threadIdx.x; c < HD; c += blockDim.x) {
        float acc = 0.f;
#pragma unroll
        for (int t = 0; t < DEC_WARPS * 4; ++t)
            if (sm_m[t] != -INFINITY) acc += sm_o[t][c] * __expf(sm_m[t] - M);
        wp[2 + c] = acc;
    }
    if (threadIdx.x == 0) {
        float L = 0.f;
#pragma unroll
        for (int t = 0; t < DEC_WARPS * 4; ++t)
            if (sm_m[t] != -INFINITY) L += sm_l[t] * __expf(sm_m[t] - M);
        wp[0] = M;
        wp[1] = L;
    }
}

template <typename T, int HD>
__global__ void attn_decode_combine_kernel(const float* __restrict__ work, int n_chunks, int len_static,
                                           const int* __restrict__ d_len_minus1, int H, T* __restrict__ o) {
    pdl_launch_dependents();
    pdl_wait();
    const int len = d_len_minus1 ? (*d_len_minus1 + 1) : len_static;
    const int used = min(n_chunks, (len + DEC_CHUNK - 1) / DEC_CHUNK);
    const int bh = blockIdx.x;
    const float* wp = work + (size_t)bh * n_chunks * (HD + 2);
    float M = -INFINITY;
    for (int c = 0; c < used; ++c) M = fmaxf(M, wp[(size_t)c * (HD + 2)]);
    for (int e = threadIdx.x; e < HD; e += blockDim.x) {
        float L = 0.f, acc = 0.f;
        for (int c = 0; c < used; ++c) {
            const float mc = wp[(size_t)c * (HD + 2)];
            if (mc == -INFINITY) continue;
            const float w = __expf(mc - M);
            L += wp[(size_t)c * (HD + 2) + 1] * w;
            acc += wp[(size_t)c * (HD + 2) + 2 + e] * w;
        }
        o[(size_t)bh * HD + e] = from_f32<T>(acc / L);
    }
}

uint64_t attention_decode_work_bytes(int B, int H, int max_len, int hd) {
    const int n_chunks = (max_len + DEC_CHUNK - 1) / DEC_CHUNK;
    return (uint64_t)B * H * n_chunks * (hd + 2) * sizeof(float);
}

template <typename T, int HD>
static int launch_dec_t(const void* q, const void* k, const void* v, void* o, int B, int H, int len,
                        const int* d_len_minus1, int kv_stride, float* work, cudaStream_t st) {
    // With a device-side length, size the grid for the largest length the
    // cache can hold; chunks past the live length exit at once.
    const int grid_len = d_len_minus1 ? kv_stride : len;
    const int n_chunks = (grid_len + DEC_CHUNK - 1) / DEC_CHUNK;
    dim3 grid(n_chunks, B * H);
    launch_pdl(attn_decode_partial_kernel<T, HD>, grid, dim3(DEC_WARPS * 32), 0, st, (const T*)q, (const T*)k,
               (const T*)v, H, len, d_len_minus1, kv_stride, 1.0f / sqrtf((float)HD), work, n_chunks);
    LLAMA_LAUNCH_CHECK();
    launch_pdl(attn_decode_combine_kernel<T, HD>, dim3(B * H), dim3(HD), 0, st, (const float*)work, n_chunks, len,
               d_len_minus1, H, (T*)o);
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}

int launch_attention_decode(int dtype, const void* q, const void* k, const void* v, void* o, int B, int H,
                            int len, const int* d_len_minus1, int hd, int kv_stride, float* work,
                            cudaStream_t st) {
    if (B <= 0) return LLAMA_OK;
#define DEC_CASE(TT, HH) return launch_dec_t<TT, HH>(q, k, v, o, B, H, len, d_len_minus1, kv_stride, work, st)
    if (dtype == LLAMA_BF16) {
        if (hd == 128) DEC_CASE(bf16, 128);
        if (hd == 64) DEC_CASE(bf16, 64);
    } else {
        if (hd == 128) DEC_CASE(float, 128);
        if (hd == 64) DEC_CASE(float, 64);
        if (hd == 32) DEC_CASE(float, 32);
    }
#undef DEC_CASE
    return LLAMA_ERR_INVALID_ARG;
}

// ---------------------------------------------------------------------------
// Decode attention with no allocation at all.
//
// Some callers cannot call cudaMalloc (or hand us an allocator) when they
// run a decode step: runtimes that plan every byte of device memory up
// front and forbid allocation once serving starts, code that must not
// allocate while it is being captured into a CUDA graph, or embedders that
// have no device allocator to give us.  For them the split-sequence
// workspace lives in a fixed array in this library's own device memory,
// loaded with the library on every GPU that uses it and held until exit.
//
// Limit: 8 MiB of workspace, i.e. B * H * ceil(len / 256) * (head_dim + 2)
// <= 2,097,152 floats (LLaMA-13B shapes at batch 32 and 2304 positions need
// 1,497,600).  Larger calls are rejected with LLAMA_ERR_OOM before anything
// is queued.  Every call shares the one array, so calls that overlap on the
// GPU (other streams, other host threads) race; each call writes every
// workspace slot it later reads, so nothing has to start at zero.
constexpr size_t NOALLOC_SCRATCH_FLOATS = (size_t)2 << 20;
static __device__ __align__(256) float g_decode_scratch[NOALLOC_SCRATCH_FLOATS];

namespace {
constexpr int MAX_DEVICES = 64;
float* g_scratch_addr[MAX_DEVICES];
std::mutex g_scratch_mu;

// Device address of the array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and kept.
int noalloc_scratch(float** out) {
    int dev = -1;
    LLAMA_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= MAX_DEVICES) return LLAMA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return LLAMA_ERR_CUDA;
        }
        g_scratch_addr[dev] = static_cast<float*>(p);
    }
    *out = g_scratch_addr[dev];
    return LLAMA_OK;
}
}  // namespace

extern "C" LLAMA_API int llama_op_attention_decode_noalloc(int32_t dtype, const void* d_q, const void* d_k,
                                                           const void* d_v, void* d_o, int32_t B, int32_t H,
                                                           int32_t len, int32_t head_dim, int32_t kv_stride,
                                                           void* stream) {
    if (!d_q || !d_k || !d_v || !d_o || B <= 0 || H <= 0 || len <= 0 || kv_stride < len)
        return LLAMA_ERR_INVALID_ARG;
    if (dtype != LLAMA_F32 && dtype != LLAMA_BF16) return LLAMA_ERR_INVALID_ARG;
    if (head_dim != 32 && head_dim != 64 && head_dim != 128) return LLAMA_ERR_INVALID_ARG;
    if (attention_decode_work_bytes(B, H, len, head_dim) > sizeof(float) * NOALLOC_SCRATCH_FLOATS)
        return LLAMA_ERR_OOM;
    float* work = nullptr;
    const int rc = noalloc_scratch(&work);
    if (rc) return rc;
    return launch_attention_decode(dtype, d_q, d_k, d_v, d_o, B, H, len, nullptr, head_dim, kv_stride, work,
                                   (cudaStream_t)stream);
}
