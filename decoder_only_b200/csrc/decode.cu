// Decode-side attention: split-sequence attention over the contiguous KV
// cache.
//
// Decode attention ("GQA Was Not an Original LLaMA Feature": every step
// reads the keys and values of all previous tokens) is HBM-bound: each
// (sequence, head) streams len * head_dim * 2 elements once.  The sequence
// is cut into chunks of 128 keys so that B*H*chunks CTAs cover the SMs; each
// chunk leaves (max, sum, unnormalised output) in the workspace, and the
// last chunk of a (sequence, head) to finish merges them (the online-softmax
// merge rule) in chunk order.
#include <mutex>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

constexpr int DEC_CHUNK = 128;   // keys per CTA: one bulk copy of K rows and one of V rows
constexpr int DEC_WARPS = 4;     // 4 warps x 4 lane groups; each group handles one key at a time

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16 bytes of T as floats
template <typename T> struct V16;
template <> struct V16<bf16> {
    static constexpr int N = 8;
    __device__ static __forceinline__ void load(const bf16* p, float* out) {
        const uint4 w = *reinterpret_cast<const uint4*>(p);
        float2 f;
        f = unpack_bf16x2(w.x); out[0] = f.x; out[1] = f.y;
        f = unpack_bf16x2(w.y); out[2] = f.x; out[3] = f.y;
        f = unpack_bf16x2(w.z); out[4] = f.x; out[5] = f.y;
        f = unpack_bf16x2(w.w); out[6] = f.x; out[7] = f.y;
    }
};
template <> struct V16<float> {
    static constexpr int N = 4;
    __device__ static __forceinline__ void load(const float* p, float* out) {
        const float4 w = *reinterpret_cast<const float4*>(p);
        out[0] = w.x; out[1] = w.y; out[2] = w.z; out[3] = w.w;
    }
};

// One CTA per (chunk of 128 keys, sequence b, head h).  The chunk's K and V
// rows are contiguous in the cache, so one bulk asynchronous copy each brings
// them to shared memory (the whole chunk is in flight at once).  Eight lanes
// share a key: lane r of a group holds dims {(u*8 + r)*VEC ..} for each
// 16-byte vector u, so a group reads 128 contiguous bytes per vector.  The
// 16 groups' (max, sum, output) merge in shared memory into the chunk's
// partial; the CTA that finishes the last chunk of (b, h) merges all chunks
// in order and writes the output row.
template <typename T, int HD>
__global__ void __launch_bounds__(DEC_WARPS * 32) attn_decode_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ o, int H, int Hkv,
    int len_static, const int* __restrict__ d_len_minus1, int kv_stride, float scale, float* __restrict__ work,
    int* __restrict__ counters, int n_chunks, int* __restrict__ err) {
    constexpr int VEC = V16<T>::N;
    constexpr int DPL = HD / 8;            // dims per lane
    constexpr int NV = DPL / VEC;          // 16-byte vectors per lane per row
    extern __shared__ __align__(128) uint8_t dsm[];
    T* sk = reinterpret_cast<T*>(dsm);                 // [DEC_CHUNK][HD]
    T* sv = sk + DEC_CHUNK * HD;                       // [DEC_CHUNK][HD]
    __shared__ __align__(8) uint64_t bar;
    __shared__ float sm_m[DEC_WARPS * 4], sm_l[DEC_WARPS * 4];
    __shared__ float sm_o[DEC_WARPS * 4][HD];
    __shared__ int last;

    pdl_launch_dependents();
    pdl_wait();   // the newest K/V row and q come from the projection before this kernel
    const int bh = blockIdx.y;
    const int b = bh / H, h = bh - b * H;
    const int len = d_len_minus1 ? (d_len_minus1[b] + 1) : len_static;   // per sequence
    const int used = (len + DEC_CHUNK - 1) / DEC_CHUNK;
    const int chunk = blockIdx.x;
    if (chunk >= used) return;                          // past the live length
    const int k_begin = chunk * DEC_CHUNK;
    const int nkeys = min(len - k_begin, DEC_CHUNK);
    const size_t head_off = ((size_t)b * Hkv + h / (H / Hkv)) * (size_t)kv_stride * HD;   // its key/value head
    const uint32_t bar_a = smem_addr(&bar);

    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_a) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        const uint32_t bytes = (uint32_t)(nkeys * HD * sizeof(T));
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_a), "r"(2 * bytes)
                     : "memory");
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                smem_addr(sk)),
            "l"(k + head_off + (size_t)k_begin * HD), "r"(bytes), "r"(bar_a)
            : "memory");
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                smem_addr(sv)),
            "l"(v + head_off + (size_t)k_begin * HD), "r"(bytes), "r"(bar_a)
            : "memory");
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 3, r = lane & 7;
    float qv[DPL];
    {
        const T* qp = q + ((size_t)b * H + h) * HD;
#pragma unroll
        for (int u = 0; u < NV; ++u) V16<T>::load(qp + (u * 8 + r) * VEC, qv + u * VEC);
#pragma unroll
        for (int e = 0; e < DPL; ++e) qv[e] *= scale;
    }
    __syncthreads();   // barrier initialised before anyone waits on it
    // bounded wait for both copies
    auto wait_copies = [bar_a](uint64_t limit_ns) {
        uint64_t t0;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
        while (true) {
            uint32_t done;
            asm volatile(
                "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}\n"
                : "=r"(done)
                : "r"(bar_a)
                : "memory");
            if (done) return true;
            uint64_t t;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
            if (t - t0 > limit_ns) return false;
        }
    };
    const bool ok = wait_copies(2000000000ull);
    if (!ok) {
        // The chunk is dropped (its partial carries no keys) and the error
        // word says so.  The copies may still be in flight into this CTA's
        // shared memory: wait for them once more (bounded) so that they do
        // not land in the next CTA placed on this SM, and read none of it.
        if (threadIdx.x == 0) atomicOr(err, LLAMA_DEVERR_TIMEOUT);
        wait_copies(2000000000ull);
    }
    float m = -INFINITY, l = 0.f, acc[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
    if (ok) {
        const int kw = warp * (DEC_CHUNK / DEC_WARPS);
#pragma unroll 2
        for (int i = 0; i < DEC_CHUNK / DEC_WARPS / 4; ++i) {
            const int j = kw + 4 * i + g;                 // key within the chunk (warp-uniform loop)
            const bool valid = j < nkeys;
            float kk[DPL], vv[DPL];
            const int jr = valid ? j : 0;
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                V16<T>::load(sk + (size_t)jr * HD + (u * 8 + r) * VEC, kk + u * VEC);
                V16<T>::load(sv + (size_t)jr * HD + (u * 8 + r) * VEC, vv + u * VEC);
            }
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) s = fmaf(qv[e], kk[e], s);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            if (valid) {
                const float m_new = fmaxf(m, s);
                const float corr = __expf(m - m_new);
                const float p = __expf(s - m_new);
                l = l * corr + p;
#pragma unroll
                for (int e = 0; e < DPL; ++e) acc[e] = fmaf(acc[e], corr, p * vv[e]);
                m = m_new;
            }
        }
    }
    // merge the 16 key groups of this chunk
    const int grp = warp * 4 + g;
    if (r == 0) {
        sm_m[grp] = m;
        sm_l[grp] = l;
    }
#pragma unroll
    for (int u = 0; u < NV; ++u)
#pragma unroll
        for (int t = 0; t < VEC; ++t) sm_o[grp][(u * 8 + r) * VEC + t] = acc[u * VEC + t];
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int t = 0; t < DEC_WARPS * 4; ++t) M = fmaxf(M, sm_m[t]);
    float* wp = work + ((size_t)bh * n_chunks + chunk) * (HD + 2);
    for (int c = threadIdx.x; c < HD; c += blockDim.x) {
        float a = 0.f;
#pragma unroll
        for (int t = 0; t < DEC_WARPS * 4; ++t)
            if (sm_m[t] != -INFINITY) a += sm_o[t][c] * __expf(sm_m[t] - M);
        wp[2 + c] = a;
    }
    if (threadIdx.x == 0) {
        float L = 0.f;
#pragma unroll
        for (int t = 0; t < DEC_WARPS * 4; ++t)
            if (sm_m[t] != -INFINITY) L += sm_l[t] * __expf(sm_m[t] - M);
        wp[0] = M;
        wp[1] = L;
    }
    // the last chunk of (b, h) to finish merges all chunks
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int prev = atomicAdd(counters + bh, 1);
        last = (prev == used - 1);
        if (last) counters[bh] = 0;   // ready for the next launch
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    const float* wb = work + (size_t)bh * n_chunks * (HD + 2);
    float Mall = -INFINITY;
    for (int c = 0; c < used; ++c) Mall = fmaxf(Mall, __ldcg(wb + (size_t)c * (HD + 2)));
    for (int e = threadIdx.x; e < HD; e += blockDim.x) {
        float L = 0.f, a = 0.f;
        for (int c = 0; c < used; ++c) {
            const float mc = __ldcg(wb + (size_t)c * (HD + 2));
            if (mc == -INFINITY) continue;
            const float w = __expf(mc - Mall);
            L += __ldcg(wb + (size_t)c * (HD + 2) + 1) * w;
            a += __ldcg(wb + (size_t)c * (HD + 2) + 2 + e) * w;
        }
        o[(size_t)bh * HD + e] = from_f32<T>(a / L);
    }
}

static size_t dec_chunks(int len) { return (size_t)(len + DEC_CHUNK - 1) / DEC_CHUNK; }

// Workspace of the standalone entry points: partials [B*H][chunks][hd + 2]
// floats, then the arrival counters [B*H] ints (the model keeps its
// counters in a buffer of their own).
static uint64_t dec_partial_bytes(int B, int H, int max_len, int hd) {
    return ((uint64_t)B * H * dec_chunks(max_len) * (hd + 2) * sizeof(float) + 15) & ~(uint64_t)15;
}

uint64_t attention_decode_work_bytes(int B, int H, int max_len, int hd) {
    return dec_partial_bytes(B, H, max_len, hd) + (uint64_t)B * H * sizeof(int);
}

int* attention_decode_counters(float* work, int B, int H, int max_len, int hd) {
    return reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(work) + dec_partial_bytes(B, H, max_len, hd));
}

template <typename T, int HD>
static int dec_attr() {
    static PerDeviceOnce once;
    return once_per_device(once, []() -> int {
        LLAMA_CUDA_TRY(cudaFuncSetAttribute(attn_decode_kernel<T, HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)(2 * (size_t)DEC_CHUNK * HD * sizeof(T))));
        return (int)LLAMA_OK;
    });
}

template <typename T, int HD>
static int launch_dec_t(const void* q, const void* k, const void* v, void* o, int B, int H, int Hkv, int len,
                        const int* d_len_minus1, int kv_stride, float* work, int* counters, int* err,
                        cudaStream_t st) {
    // With a device-side length the grid covers every chunk the cache can
    // hold; chunks past the live length exit at once.
    const int grid_len = d_len_minus1 ? kv_stride : len;
    const int n_chunks = (int)dec_chunks(grid_len);
    const size_t smem = 2 * (size_t)DEC_CHUNK * HD * sizeof(T);
    int rc = dec_attr<T, HD>();
    if (rc) return rc;
    launch_pdl(attn_decode_kernel<T, HD>, dim3(n_chunks, B * H), dim3(DEC_WARPS * 32), smem, st, (const T*)q,
               (const T*)k, (const T*)v, (T*)o, H, Hkv, len, d_len_minus1, kv_stride, 1.0f / sqrtf((float)HD), work,
               counters, n_chunks, err);
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}

// Sets the shared-memory attribute of every instantiation (before any capture).
int attention_decode_prepare() {
    int rc;
    if ((rc = dec_attr<bf16, 128>()) || (rc = dec_attr<bf16, 64>()) || (rc = dec_attr<float, 128>()) ||
        (rc = dec_attr<float, 64>()))
        return rc;
    return dec_attr<float, 32>();
}

// Zeroes the arrival counters of a standalone workspace (the model zeroes
// its own once; every launch leaves them at zero).
int attention_decode_clear(float* work, int B, int H, int len, int hd, cudaStream_t st) {
    LLAMA_CUDA_TRY(cudaMemsetAsync(attention_decode_counters(work, B, H, len, hd), 0, (size_t)B * H * sizeof(int),
                                   st));
    return LLAMA_OK;
}

int launch_attention_decode(int dtype, const void* q, const void* k, const void* v, void* o, int B, int H,
                            int Hkv, int len, const int* d_len_minus1, int hd, int kv_stride, float* work,
                            int* counters, int* err, cudaStream_t st) {
    if (B <= 0) return LLAMA_OK;
    if (Hkv <= 0 || H % Hkv != 0) return LLAMA_ERR_INVALID_ARG;
#define DEC_CASE(TT, HH) \
    return launch_dec_t<TT, HH>(q, k, v, o, B, H, Hkv, len, d_len_minus1, kv_stride, work, counters, err, st)
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
// Limit: 8 MiB of workspace, i.e. B * H * ceil(len / 128) * (head_dim + 2)
// floats plus B * H arrival counters (LLaMA-13B shapes at batch 32 and 2304
// positions need about 11.5 MB -- larger than the limit -- so that case
// goes through the workspace entry point; LLaMA-7B shapes at batch 4 need
// 1.2 MB).  Larger calls are rejected with LLAMA_ERR_OOM before anything is
// queued.  Every call shares the one array, so calls that overlap on the
// GPU (other streams, other host threads) race.  The arrival counters must
// start at zero: each call clears them before its kernel runs; every other
// slot a call reads, it writes first.
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
    int rc = noalloc_scratch(&work);
    if (rc) return rc;
    int* err = nullptr;
    if ((rc = op_error_word(&err))) return rc;
    if ((rc = attention_decode_clear(work, B, H, len, head_dim, (cudaStream_t)stream))) return rc;
    return launch_attention_decode(dtype, d_q, d_k, d_v, d_o, B, H, H, len, nullptr, head_dim, kv_stride, work,
                                   attention_decode_counters(work, B, H, len, head_dim), err, (cudaStream_t)stream);
}
