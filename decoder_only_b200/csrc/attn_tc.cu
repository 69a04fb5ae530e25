// Causal flash attention for prefill on the sm_100a tensor cores.
//
// Per head: O = softmax(Q K^T / sqrt(hd) + causal mask) V ("LLaMA is a pull
// request against the 2017 transformer": attention untouched, causal mask;
// "RoPE: rotate Q and K, leave V alone": Q and K arrive rotated).  The
// fully masked key tiles above the diagonal are never computed, and the
// (S x S) score matrix is never written to memory -- the two ideas the
// knowledge note credits to the xFormers attention of the training system.
//
// Persistent CTAs, one per SM, each working through a list of work items
// (128-query tile, head, sequence): longest items first, dealt in snake
// order.  The tile rings and barriers run on over item boundaries, so the
// next item's Q, K and first scores load and compute while the current
// item's output is written.
//   warp 0      TMA: lane 0 each item's Q (once the previous item's last
//               Q K^T is done), then its K_j tiles; lane 1 the V_j tiles
//               (2-stage rings; K_j is free once S_j is computed, V_j once
//               O_j is, so K runs ahead of V).  3-D tensor maps (hd,
//               position, head) make rows >= S read as 0.
//   warp 1      TMEM allocator + MMA issuer:
//                 S_j = Q K_j^T        (M 128, N 128, K hd)  -> TMEM S[j % 2]
//                 O  += P_j V_j        (M 128, N hd, K 128)  -> TMEM O (one
//                                       accumulator for the whole row tile)
//               V is the MN-major B operand (hd contiguous), so the cache
//               layout [position][hd] is used as is.
//   warps 2..5  one query row per thread: row max of S_j (pass 1), then
//               p = 2^(s log2e / sqrt(hd) - m) rounded to bf16 into the
//               shared P tile (128-byte swizzled, K-major) and the row sum
//               (pass 2), both passes on the row's 128 scores held in
//               registers (one TMEM read per tile).  The running maximum m
//               (log2 units) moves only when a tile's maximum exceeds it by
//               more than 8: p stays <= 2^8, exact in fp32 and bf16's range,
//               and the output in TMEM is rescaled by 2^(m_old - m_new) (TMEM
//               load, scale, store, after the previous P V product) only
//               then -- a few times per row -- instead of folding every
//               tile's product into registers.  The pass is bound by the
//               instructions it issues per score (one warp per sub-
//               partition): one FMA, one ex2, half a pack, one add.
//               After an item's last tile: O / (row sum), bf16, to
//               global; the item's first P V product waits for that read.
// All mbarrier waits are bounded (see tcgen05.cuh).
#include <cudaTypedefs.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace {

using namespace tc;

constexpr int BQ = 128;         // queries per tile
constexpr int BKV = 128;        // keys per tile
constexpr int NTHREADS = 192;
constexpr float RESCALE_LOG2 = 8.f;   // move the running maximum only by more than this (log2 units)

// 2^x by the special-function unit's approximation (one instruction;
// relative error far below bf16's 2^-9; 2^-inf = 0 for masked scores)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int HD>
struct ACfg {
    static constexpr int REG = 128 * 128;                    // one [128 rows][64 bf16] swizzled region, bytes
    static constexpr int NREG = HD / 64;                     // regions per Q / K / V tile
    static constexpr int TILE = NREG * REG;                  // Q, K or V tile bytes
    static constexpr int P_TILE = 2 * REG;                   // P: [128 q][128 keys] bf16
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + TILE;               // [2]
    static constexpr int OFF_V = OFF_K + 2 * TILE;           // [2]
    static constexpr int OFF_P = OFF_V + 2 * TILE;           // [2]
    static constexpr int OFF_BAR = OFF_P + 2 * P_TILE;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;               // S[2] at 0, 128; O at 256
};

// P tile position of 8 consecutive keys (one 16-byte chunk) of query row t:
// region by key half, 128-byte row t, chunk index XOR (t % 8).
__device__ __forceinline__ uint32_t p_chunk_addr(uint32_t base, int t, int chunk16) {
    const int region = chunk16 >> 3;
    const int c = chunk16 & 7;
    return base + region * (128 * 128) + t * 128 + ((c ^ (t & 7)) << 4);
}

template <int HD>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, bf16* __restrict__ out, int H, int S,
                           int Hkv, int B, float scale_log2, const int* __restrict__ pages, int pps, int* err) {
    using C = ACfg<HD>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t sQ = base + C::OFF_Q, sK = base + C::OFF_K, sV = base + C::OFF_V, sP = base + C::OFF_P;
    const uint32_t bars = base + C::OFF_BAR;
    const uint32_t q_full = bars;
    const uint32_t k_full = bars + 8;        // [2]
    const uint32_t v_full = bars + 24;       // [2]
    const uint32_t k_empty = bars + 40;      // [2]
    const uint32_t s_full = bars + 56;       // [2]
    const uint32_t s_empty = bars + 72;      // [2]
    const uint32_t p_full = bars + 88;       // [2]
    const uint32_t o_done = bars + 104;      // one phase per completed P V product
    const uint32_t o_last = bars + 112;      // one phase per work item: its last P V product
    const uint32_t q_empty = bars + 120;     // one phase per work item: its last Q K^T (Q free)
    const uint32_t o_free = bars + 128;      // one phase per work item: its output read out of TMEM
    const uint32_t v_empty = bars + 136;     // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_BAR + 160);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    // Work items (128-query tile, head, sequence), longest (most key tiles)
    // first, dealt to the persistent CTAs in snake order (CTA c takes item
    // c of the first G, item 2G - 1 - c of the next G, ...), which evens out
    // the CTAs' key-tile totals.  Per-tile rings run on counters over all of
    // a CTA's items, so one item's start overlaps the previous one's end.
    const int n_qt = (S + BQ - 1) / BQ;
    const int total = n_qt * H * B;
    const int G = (int)gridDim.x, cta = (int)blockIdx.x;
    auto item_at = [&](int n) { return n * G + ((n & 1) ? G - 1 - cta : cta); };
    auto item = [&](int it, int& qt, int& h, int& b) {
        qt = n_qt - 1 - it / (H * B);
        const int r = it - (n_qt - 1 - qt) * (H * B);
        h = r % H;
        b = r / H;
    };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(k_full + 8 * i, 1);
            mbar_init(v_full + 8 * i, 1);
            mbar_init(k_empty + 8 * i, 1);
            mbar_init(v_empty + 8 * i, 1);
            mbar_init(s_full + 8 * i, 1);
            mbar_init(s_empty + 8 * i, 128);
            mbar_init(p_full + 8 * i, 128);
        }
        mbar_init(o_done, 1);
        mbar_init(o_last, 1);
        mbar_init(q_empty, 1);
        mbar_init(o_free, 128);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();   // Q, K, V come from the projection kernel before this one

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane < 2) {
            // lane 0: each item's Q (once the previous item's last Q K^T is done), then its K_j;
            // lane 1: the V_j
            const bool is_k = (lane == 0);
            const uint32_t full = is_k ? k_full : v_full, empty = is_k ? k_empty : v_empty;
            const uint32_t dst = is_k ? sK : sV;
            const CUtensorMap* map = is_k ? &tmK : &tmV;
            bool ok = true;
            int kt = 0, ni = 0, q_loads = 0;
            for (int it = item_at(0); it < total && ok; it = item_at(++ni)) {
                int qt, h, b;
                item(it, qt, h, b);
                const int kv_head = b * Hkv + h / (H / Hkv);      // grouped keys and values
                if (is_k) {
                    if (ni > 0 && !mbar_wait(q_empty, (uint32_t)((ni - 1) & 1), abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(q_full, C::TILE);
                    for (int r = 0; r < C::NREG; ++r)
                        tma_load_3d(sQ + r * C::REG, &tmQ, q_full, 64 * r, qt * BQ, b * H + h);
                    ++q_loads;
                }
                for (int j = 0; j <= qt; ++j, ++kt) {
                    const int st = kt & 1;
                    if (!mbar_wait(empty + 8 * st, ((kt >> 1) & 1) ^ 1u, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(full + 8 * st, C::TILE);
                    for (int r = 0; r < C::NREG; ++r)
                        // paged cache: key tile j is page pages[b][j] (KV_PAGE == BKV positions)
                        tma_load_3d(dst + st * C::TILE + r * C::REG, map, full + 8 * st, 64 * r, pages ? 0 : j * BKV,
                                    pages ? __ldg(pages + b * pps + j) * Hkv + (kv_head - b * Hkv) : kv_head);
                }
            }
            if (!ok) {
                // drain (bounded) the copies this thread issued
                const uint64_t t0 = global_timer();
                while (is_k && q_loads > 0 && !mbar_try_wait(q_full, (uint32_t)((q_loads - 1) & 1)) &&
                       global_timer() - t0 < WAIT_LIMIT_NS / 4) {
                }
                for (int t = kt > 2 ? kt - 2 : 0; t < kt; ++t) {
                    const uint32_t par = (t >> 1) & 1;
                    while (!mbar_try_wait(full + 8 * (t & 1), par) && global_timer() - t0 < WAIT_LIMIT_NS / 2) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_QK = idesc_bf16(BKV);                 // K-major A and B
            constexpr uint32_t IDESC_PV = idesc_bf16(HD) | (1u << 16);      // B (V) MN-major
            bool ok = true;
            int kt0 = 0, ni = 0;
            for (int it = item_at(0); it < total && ok; it = item_at(++ni)) {
                int qt, h, b;
                item(it, qt, h, b);
                const int n_kv = qt + 1;
                ok = mbar_wait(q_full, (uint32_t)(ni & 1), abort_flag, err);
                tc_fence_after();
                for (int j = 0; j <= n_kv && ok; ++j) {
                    if (j < n_kv) {
                        const int t = kt0 + j, st = t & 1;
                        const uint32_t par = (t >> 1) & 1;
                        if (!mbar_wait(k_full + 8 * st, par, abort_flag, err) ||
                            !mbar_wait(s_empty + 8 * st, par ^ 1u, abort_flag, err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d_s = tmem + (uint32_t)(st * 128);
#pragma unroll
                        for (int kk = 0; kk < HD / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * C::REG + (kk & 3) * 32;
                            umma_bf16(d_s, sw128_desc(sQ + off), sw128_desc(sK + st * C::TILE + off), IDESC_QK,
                                      kk > 0 ? 1u : 0u);
                        }
                        umma_commit(s_full + 8 * st);
                        umma_commit(k_empty + 8 * st);
                        if (j == n_kv - 1) umma_commit(q_empty);   // Q free for the next item
                    }
                    if (j > 0) {
                        // P_jj is complete (and O rescaled where a row's maximum moved)
                        const int jj = j - 1, t = kt0 + jj, st = t & 1;
                        const uint32_t par = (t >> 1) & 1;
                        if (!mbar_wait(p_full + 8 * st, par, abort_flag, err) ||
                            !mbar_wait(v_full + 8 * st, par, abort_flag, err) ||
                            (jj == 0 && ni > 0 && !mbar_wait(o_free, (uint32_t)((ni - 1) & 1), abort_flag, err))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d_o = tmem + 256u;
#pragma unroll
                        for (int kk = 0; kk < BKV / 16; ++kk) {
                            // A = P (K-major, keys contiguous); B = V (MN-major): 16 keys = 2 groups of 8 rows
                            const uint32_t poff = (kk >> 2) * C::REG + (kk & 3) * 32;
                            uint64_t vd = sw128_desc(sV + st * C::TILE + kk * 2048);
                            vd = (vd & ~(((uint64_t)0x3FFF) << 16)) | ((uint64_t)(C::REG >> 4) << 16);   // LBO: next 64 hd
                            umma_bf16(d_o, sw128_desc(sP + st * C::P_TILE + poff), vd, IDESC_PV,
                                      (jj > 0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit(o_done);
                        umma_commit(v_empty + 8 * st);
                        if (jj == n_kv - 1) umma_commit(o_last);
                    }
                }
                kt0 += n_kv;
            }
        }
    } else {
        // ---------------------------------------------------------- softmax + output (warps 2..5)
        const int quarter = warp & 3;
        const int t_row = quarter * 32 + lane;           // query row within the tile
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const uint32_t o_addr = tmem + lane_addr + 256u;
        bool ok = true;
        int kt0 = 0, ni = 0;
        for (int it = item_at(0); it < total && ok; it = item_at(++ni)) {
            int qt, h, b;
            item(it, qt, h, b);
            const int n_kv = qt + 1;
            const int q = qt * BQ + t_row;
            float m = -INFINITY, l = 0.f;                // running maximum (log2 units) and row sum
            for (int j = 0; j < n_kv; ++j) {
                const int t = kt0 + j, st = t & 1;
                const uint32_t par = (t >> 1) & 1;
                // warp-uniform decision: the TMEM loads below are warp-collective
                if (!__all_sync(0xffffffffu, mbar_wait(s_full + 8 * st, par, abort_flag, err))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t s_addr = tmem + lane_addr + (uint32_t)(st * 128);
                // the row's 128 scores, four TMEM loads in flight, one wait
                float sv[128];
                {
                    uint32_t* r = reinterpret_cast<uint32_t*>(sv);
#pragma unroll
                    for (int c = 0; c < 4; ++c) TMEM_LD_X32(s_addr + c * 32, (r + 32 * c));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                }
                // only the diagonal tile masks: there key k is visible iff
                // k <= min(q, S - 1) (a select per score, no branch)
                if (j == n_kv - 1) {
                    const int lim = min(q, S - 1) - j * BKV;
#pragma unroll
                    for (int i = 0; i < 128; ++i) sv[i] = (i <= lim) ? sv[i] : -INFINITY;
                }
                // pass 1: row maximum, eight independent partial maxima
                float mx8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) mx8[u] = sv[u];
#pragma unroll
                for (int i = 8; i < 128; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], sv[i]);
                const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
                // the running maximum moves (and O is rescaled) only by more than RESCALE_LOG2
                const float mt = mx * scale_log2;
                float corr = 1.f;
                bool rescale = false;
                if (m == -INFINITY) {
                    m = mt;                              // first tile: nothing accumulated yet
                } else if (mt > m + RESCALE_LOG2) {
                    corr = ex2_approx(m - mt);
                    m = mt;
                    rescale = true;
                }
                // pass 2: probabilities (bf16) into the P tile; the row sum adds
                // the fp32 values in four independent partial sums
                float rs4[4] = {0.f, 0.f, 0.f, 0.f};
                const uint32_t pbase = sP + st * C::P_TILE;
#pragma unroll
                for (int c = 0; c < 16; ++c) {           // 16 chunks of 8 keys (16 bytes of P)
                    uint32_t pk[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float p0 = ex2_approx(fmaf(sv[8 * c + 2 * i], scale_log2, -m));
                        const float p1 = ex2_approx(fmaf(sv[8 * c + 2 * i + 1], scale_log2, -m));
                        pk[i] = pack_bf16x2(p0, p1);
                        rs4[i] += p0 + p1;
                    }
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(p_chunk_addr(pbase, t_row, c)),
                                 "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3])
                                 : "memory");
                }
                const float rs = (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
                tc_fence_before();
                mbar_arrive(s_empty + 8 * st);
                // a warp with a moved maximum rescales its 32 rows of O once the
                // previous P V product is done.  Its completion is phase t - 1 of
                // o_done: S_t's completion (waited for above) follows that of
                // P_{t-2} V_{t-2}, and P_t V_t waits for this warp, so the
                // barrier is in phase t - 1 or t here.
                if (__any_sync(0xffffffffu, rescale)) {
                    bool w = mbar_wait(o_done, (uint32_t)((t - 1) & 1), abort_flag, err);
                    if (!__all_sync(0xffffffffu, w)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < HD / 32; ++c) {
                        float ov[32];
                        tmem_ld32(o_addr + c * 32, ov);
#pragma unroll
                        for (int i = 0; i < 32; ++i) ov[i] *= corr;
                        tmem_st32(o_addr + c * 32, ov);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                }
                l = l * corr + rs;
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(p_full + 8 * st);
            }
            // the item's last product: O / l, bf16, to global; then O is free for the next item
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_last, (uint32_t)(ni & 1), abort_flag, err));
            if (!ok) break;
            tc_fence_after();
            const float inv = 1.f / l;
            bf16* dst = out + ((size_t)b * S + q) * ((size_t)H * HD) + (size_t)h * HD;
#pragma unroll 1
            for (int c = 0; c < HD / 32; ++c) {
                float ov[32];
                tmem_ld32(o_addr + c * 32, ov);
                if (q < S) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint4 w = make_uint4(pack_bf16x2(ov[8 * u] * inv, ov[8 * u + 1] * inv),
                                             pack_bf16x2(ov[8 * u + 2] * inv, ov[8 * u + 3] * inv),
                                             pack_bf16x2(ov[8 * u + 4] * inv, ov[8 * u + 5] * inv),
                                             pack_bf16x2(ov[8 * u + 6] * inv, ov[8 * u + 7] * inv));
                        *reinterpret_cast<uint4*>(dst + c * 32 + 8 * u) = w;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(o_free);
            kt0 += n_kv;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                     : "memory");
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_attn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 3-D map over [heads][rows][hd] bf16 with `rows` valid rows per head
// (rows past them read as zero), `stride_rows` rows apart; box (64, 128, 1).
int make_head_map(CUtensorMap* map, const void* ptr, int hd, int rows, int stride_rows, int heads) {
    auto fn = encode_fn_attn();
    if (!fn) return LLAMA_ERR_CUDA;
    cuuint64_t dims[3] = {(cuuint64_t)hd, (cuuint64_t)rows, (cuuint64_t)heads};
    cuuint64_t strides[2] = {(cuuint64_t)hd * 2, (cuuint64_t)stride_rows * hd * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? LLAMA_OK : LLAMA_ERR_CUDA;
}

template <int HD>
int attn_attr() {
    static PerDeviceOnce once;
    return once_per_device(once, []() -> int {
        LLAMA_CUDA_TRY(cudaFuncSetAttribute(attn_prefill_tc_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            ACfg<HD>::SMEM));
        return (int)LLAMA_OK;
    });
}

}  // namespace

int attention_tc_prepare() {
    if (!encode_fn_attn()) return LLAMA_ERR_CUDA;
    int rc = attn_attr<128>();
    if (rc) return rc;
    return attn_attr<64>();
}

int launch_attention_prefill_tc(const void* q, const void* k, const void* v, void* o, int B, int H, int Hkv, int S,
                                int hd, int kv_stride, int* err, cudaStream_t st, const int* pages, int pps,
                                int n_pages) {
    if (B <= 0 || S <= 0) return LLAMA_OK;
    if (hd != 64 && hd != 128) return LLAMA_ERR_INVALID_ARG;
    if (Hkv <= 0 || H % Hkv != 0) return LLAMA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
         reinterpret_cast<uintptr_t>(o)) & 15u)
        return LLAMA_ERR_INVALID_ARG;
    CUtensorMap mq, mk, mv;
    int rc;
    if ((rc = make_head_map(&mq, q, hd, S, S, B * H))) return rc;
    if (pages) {
        // the page pool [page][Hkv][KV_PAGE][hd]: one (page, head) slab per z coordinate
        static_assert(KV_PAGE == BKV, "a key tile is one page");
        if ((rc = make_head_map(&mk, k, hd, KV_PAGE, KV_PAGE, n_pages * Hkv))) return rc;
        if ((rc = make_head_map(&mv, v, hd, KV_PAGE, KV_PAGE, n_pages * Hkv))) return rc;
    } else {
        if ((rc = make_head_map(&mk, k, hd, S, kv_stride, B * Hkv))) return rc;
        if ((rc = make_head_map(&mv, v, hd, S, kv_stride, B * Hkv))) return rc;
    }
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)hd);
    // persistent CTAs: one per SM (or per work item, if fewer)
    const int items = ((S + BQ - 1) / BQ) * H * B;
    static int n_sm = 0;
    if (!n_sm) n_sm = tc_num_sms();
    dim3 grid(items < n_sm ? items : n_sm);
    if (hd == 128) {
        if ((rc = attn_attr<128>())) return rc;
        launch_pdl(attn_prefill_tc_kernel<128>, grid, dim3(NTHREADS), ACfg<128>::SMEM, st, mq, mk, mv, (bf16*)o, H, S,
                   Hkv, B, scale_log2, pages, pps, err);
    } else {
        if ((rc = attn_attr<64>())) return rc;
        launch_pdl(attn_prefill_tc_kernel<64>, grid, dim3(NTHREADS), ACfg<64>::SMEM, st, mq, mk, mv, (bf16*)o, H, S,
                   Hkv, B, scale_log2, pages, pps, err);
    }
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}
