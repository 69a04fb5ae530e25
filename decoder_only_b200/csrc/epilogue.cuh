// Epilogues applied to 32 consecutive output columns of one GEMM row.
//
// One implementation of each step, called from the tensor-core GEMM's
// fused epilogue (values straight from TMEM), from the fp32 SIMT path and
// from the decode split-K reduction.
//
//   EPI_F32     logits / plain store:       out[m, n] = acc
//   EPI_RESID   residual add into the trunk: trunk[m, n] += acc
//               ("The one formula": the skip link adds, never rescales)
//   EPI_SWIGLU  act[m, j] = SiLU(gate_j) * up_j, gate/up columns interleaved
//               in blocks of 128 (SwiGLU section; SiLU(u) = u / (1 + e^-u))
//   EPI_QKV     split [Q K V] columns, rotate Q and K per head with RoPE
//               (pair (2i, 2i+1) by pos * theta^(-2i/hd), cos/sin table
//               built in fp64 on the host), write Q and append K, V to the
//               cache ("RoPE: rotate Q and K, leave V alone").
#pragma once

#include "common.cuh"

enum EpiMode { EPI_F32 = 0, EPI_RESID = 1, EPI_SWIGLU = 2, EPI_QKV = 3 };

struct EpiArgs {
    int M, N;             // logical output rows (tokens) and columns
    float* out;           // EPI_F32 / EPI_RESID: fp32 [M, ld_out]
    int ld_out;
    float* partial;       // decode split-K workspace: fp32 [splits][M][N]
    int* counters;        // decode split-K arrival counters (zero between launches)
    void* act;            // EPI_SWIGLU: T [M, hidden]
    int hidden;
    void* q;              // EPI_QKV: T [B][H][S][hd]  (decode: [B][H][1][hd])
    void* kc;             // EPI_QKV: this layer's K cache T [B][H][smax][hd]
    void* vc;             //          and V cache
    const float2* rope;   // [max_seq][hd/2] (cos, sin)
    const int* d_pos;     // decode: position of each sequence (device, [B]); NULL in prefill
    int S;                // tokens per sequence in this call (prefill), 1 in decode
    int H, hd, d, smax;
    int Hkv;              // key/value heads: columns [d, d + Hkv hd) are K, then V
    const float* bias;    // the bias variant: fp32 per output column (weight row order), or NULL
    int m0;               // EPI_QKV prefill: token row of the GEMM's first row (row blocks launched apart)
    const int* pages;     // paged KV cache: page of (sequence b, logical page p) at pages[b * pps + p],
    int pps;              // a page holding KV_PAGE positions of every key/value head; NULL: contiguous
};

constexpr int KV_PAGE = 128;   // positions per page of a paged KV cache

// Element offset of cache row (sequence b, key/value head kvh, position pos):
// contiguous [B][Hkv][smax][hd], or paged [page][Hkv][KV_PAGE][hd]
__host__ __device__ __forceinline__ size_t kv_row_offset(const int* pages, int pps, int b, int Hkv, int kvh, int smax,
                                                         int pos, int hd) {
    if (pages) {
        const int pg = pages[b * pps + pos / KV_PAGE];
        return (((size_t)pg * Hkv + kvh) * KV_PAGE + pos % KV_PAGE) * hd;
    }
    return (((size_t)b * Hkv + kvh) * smax + pos) * hd;
}

__device__ __forceinline__ float silu_f(float u) { return u / (1.0f + __expf(-u)); }

template <typename T>
__device__ __forceinline__ void store32(T* dst, const float (&v)[32]);

template <>
__device__ __forceinline__ void store32<float>(float* dst, const float (&v)[32]) {
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int j = 0; j < 8; ++j) d4[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}

template <>
__device__ __forceinline__ void store32<bf16>(bf16* dst, const float (&v)[32]) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        d4[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                           pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
}

// 32 bias values starting at column n0 (zeros without the bias variant)
__device__ __forceinline__ void bias32(const float* bias, int n0, float (&b)[32]) {
    if (bias) {
        const float4* p = reinterpret_cast<const float4*>(bias + n0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 t = p[j];
            b[4 * j] = t.x;
            b[4 * j + 1] = t.y;
            b[4 * j + 2] = t.z;
            b[4 * j + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) b[j] = 0.f;
    }
}

// Residual add of 32 columns (n0 % 32 == 0, n0 + 32 <= N), plus the bias.
__device__ __forceinline__ void epi_resid32(const EpiArgs& a, int m, int n0, const float (&v)[32]) {
    float4* p = reinterpret_cast<float4*>(a.out + (size_t)m * a.ld_out + n0);
    float b[32];
    bias32(a.bias, n0, b);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float4 t = p[j];
        t.x += v[4 * j] + b[4 * j];
        t.y += v[4 * j + 1] + b[4 * j + 1];
        t.z += v[4 * j + 2] + b[4 * j + 2];
        t.w += v[4 * j + 3] + b[4 * j + 3];
        p[j] = t;
    }
}

// Plain fp32 store of up to 32 columns (masked at N).
__device__ __forceinline__ void epi_f32_32(const EpiArgs& a, int m, int n0, const float (&v)[32]) {
    float* p = a.out + (size_t)m * a.ld_out + n0;
    if (n0 + 32 <= a.N && (a.ld_out % 4) == 0) {
        store32<float>(p, v);
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (n0 + j < a.N) p[j] = v[j];
    }
}

// SwiGLU: hidden units j0..j0+31 from their gate and up pre-activations
// (weight rows (j0 / 128) * 256 + j0 % 128 .. and 128 rows further).
template <typename T>
__device__ __forceinline__ void epi_swiglu32(const EpiArgs& a, int m, int j0, const float (&g)[32],
                                             const float (&u)[32]) {
    const int ng = (j0 / 128) * 256 + (j0 % 128);
    float bg[32], bu[32];
    bias32(a.bias, ng, bg);
    bias32(a.bias, ng + 128, bu);
    float r[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) r[j] = silu_f(g[j] + bg[j]) * (u[j] + bu[j]);
    store32<T>(reinterpret_cast<T*>(a.act) + (size_t)m * a.hidden + j0, r);
}

// Q/K/V split + RoPE + KV-cache append for columns n0..n0+31 of token row m.
// Columns: Q [0, d), K [d, d + kvd), V [d + kvd, d + 2 kvd), kvd = Hkv * hd.
template <typename T>
__device__ __forceinline__ void epi_qkv32(const EpiArgs& a, int m, int n0, const float (&v)[32]) {
    const int kvd = a.Hkv * a.hd;
    const int which = n0 < a.d ? 0 : (n0 < a.d + kvd ? 1 : 2);   // 0 = Q, 1 = K, 2 = V
    const int c = which == 0 ? n0 : n0 - a.d - (which - 1) * kvd;
    const int head = c / a.hd;           // query head (Q) or key/value head (K, V)
    const int i0 = c - head * a.hd;      // multiple of 32 within the head
    float bq[32];
    bias32(a.bias, n0, bq);
    int b, s, pos;
    if (a.d_pos) {                       // decode: one token per sequence at its own position
        b = m;
        s = 0;
        pos = a.d_pos[m];
    } else {
        b = (m + a.m0) / a.S;
        s = (m + a.m0) - b * a.S;
        pos = s;
    }
    float r[32];
    if (which < 2) {
        const float2* cs = a.rope + (size_t)pos * (a.hd / 2) + i0 / 2;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            float2 t = cs[j];
            float x0 = v[2 * j] + bq[2 * j], x1 = v[2 * j + 1] + bq[2 * j + 1];
            r[2 * j] = x0 * t.x - x1 * t.y;
            r[2 * j + 1] = x0 * t.y + x1 * t.x;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = v[j] + bq[j];
    }
    T* dst;
    if (which == 0) {
        dst = reinterpret_cast<T*>(a.q) + (((size_t)b * a.H + head) * a.S + s) * a.hd + i0;
    } else {
        T* base = reinterpret_cast<T*>(which == 1 ? a.kc : a.vc);
        dst = base + kv_row_offset(a.pages, a.pps, b, a.Hkv, head, a.smax, pos, a.hd) + i0;
    }
    store32<T>(dst, r);
}
