// bf16 tensor-core GEMM for sm_100a: tcgen05.mma with fp32 accumulators in
// tensor memory, operands staged by TMA, fused epilogues.
//
// Computes D[r, c] = sum_k A[r, k] * B[c, k] for the projections of the
// block ("The one formula"): Q/K/V (+RoPE), O (+residual), gate/up
// (+SwiGLU), down (+residual) and the output head.  Both operands are
// K-major bf16; A supplies the 128 rows that map onto the 128 TMEM lanes.
//
//   prefill (swap = 0): A = activations [tokens, K], B = weights [N, K],
//                       tile 128 x 256, fused epilogue on the output tile.
//   (the decode projections, with the batch as N, run inside the fused
//   decode step of decode_step.cu)
//
// Warp roles (192 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer (one elected lane): stage ring of S slots
//   warp 1      TMEM allocator + MMA issuer (one lane): 4 x K=16 per stage
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 32 columns per warp,
//               TMEM accumulators double-buffered so the epilogue of
//               tile i overlaps the mainloop of tile i+1.
// Every mbarrier wait is bounded (~2 s); on expiry the CTA records
// LLAMA_DEVERR_TIMEOUT in the error word, drains its own TMA copies, frees
// its TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace {

using namespace tc;

constexpr int BM = 128;
constexpr int BK = 64;                 // 64 bf16 = one 128-byte swizzle row
constexpr int NTHREADS = 192;
template <int BN>
struct Cfg {
    static constexpr int A_BYTES = BM * BK * 2;            // 16 KB
    static constexpr int B_BYTES = BN * BK * 2;            // BN * 128 B
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = 4;
    static constexpr int TMEM_COLS = 2 * BN;                          // two accumulators
    static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
};

struct TileSched {
    int m_blocks, n_blocks, splits, kb_total, group;
    int skip_first_load;   // test hook: leave the first activation tile unrequested (its wait must expire)
    __device__ __forceinline__ int num_tiles() const { return m_blocks * n_blocks * splits; }
    // prefill: grouped raster (group m-blocks, n fastest inside a group); decode: m fastest
    __device__ __forceinline__ void get(int t, int& mb, int& nb, int& sp, int& kb0, int& kb1) const {
        if (splits > 1 || n_blocks == 1) {
            mb = t % m_blocks;
            const int rest = t / m_blocks;
            nb = rest % n_blocks;
            sp = rest / n_blocks;
        } else {
            const int per_group = group * n_blocks;
            const int g = t / per_group;
            const int w = t - g * per_group;
            const int gm = min(group, m_blocks - g * group);
            mb = g * group + w % gm;
            nb = w / gm;
            sp = 0;
        }
        const int per = (kb_total + splits - 1) / splits;
        kb0 = sp * per;
        kb1 = min(kb_total, kb0 + per);
    }
};

template <int BN, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TileSched ts,
                   EpiArgs ep, int* err) {
    using C = Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t sA = base;                                   // STAGES x A tile
    const uint32_t sB = base + C::STAGES * C::A_BYTES;          // STAGES x B tile
    const uint32_t bars = base + C::STAGES * C::STAGE_BYTES;    // barrier block
    const uint32_t full_bar = bars;                             // [STAGES]
    const uint32_t empty_bar = bars + 8 * C::STAGES;            // [STAGES]
    const uint32_t tfull_bar = bars + 16 * C::STAGES;           // [2]
    const uint32_t tempty_bar = tfull_bar + 16;                 // [2]
    const uint32_t drain_bar = tfull_bar + 48;                  // the MMA issuer's last commit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::STAGES * C::STAGE_BYTES + 16 * C::STAGES + 32);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);


    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full_bar + 8 * s, 1);
            mbar_init(empty_bar + 8 * s, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(tfull_bar + 8 * i, 1);
            mbar_init(tempty_bar + 8 * i, 128);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
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
    const uint32_t tmem_base = *tmem_slot;
    const int n_tiles = ts.num_tiles();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        // The weight operand (B) does not depend on the kernels before this
        // one: the weight tiles of the first stages are requested before
        // waiting for the predecessor, the activation tiles after it.
        if (lane == 0) {
            const CUtensorMap* w_map = &tmB;     // weights
            const CUtensorMap* x_map = &tmA;     // activations
            const uint32_t w_base = sB;
            const uint32_t x_base = sA;
            const int w_bytes = C::B_BYTES;
            const int x_bytes = C::A_BYTES;
            int stage = 0;
            uint32_t phase = 0;
            uint32_t filled = 0, fill_phase = 0;   // per-stage: filled at least once / parity of last fill
            bool ok = true;
            int pre = 0;                           // k-blocks of the first tile whose weights are in flight
            if ((int)blockIdx.x < n_tiles) {
                int mb, nb, sp, kb0, kb1;
                ts.get(blockIdx.x, mb, nb, sp, kb0, kb1);
                pre = min(C::STAGES, kb1 - kb0);
                const int w_row = nb * BN;
                for (int i = 0; i < pre; ++i) {    // fresh ring: every stage starts empty
                    mbar_expect_tx(full_bar + 8 * i, C::STAGE_BYTES);
                    tma_load_2d(w_base + i * w_bytes, w_map, full_bar + 8 * i, (kb0 + i) * BK, w_row);
                    filled |= 1u << i;
                }
            }
            pdl_wait();
            int it = 0;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
                int mb, nb, sp, kb0, kb1;
                ts.get(t, mb, nb, sp, kb0, kb1);
                const int w_row = nb * BN;
                const int x_row = mb * BM;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    if (it >= pre) {
                        if (!mbar_wait(empty_bar + 8 * stage, phase ^ 1u, abort_flag, err)) {
                            ok = false;
                            break;
                        }
                        mbar_expect_tx(full_bar + 8 * stage, C::STAGE_BYTES);
                        tma_load_2d(w_base + stage * w_bytes, w_map, full_bar + 8 * stage, kb * BK, w_row);
                    }
                    if (!(ts.skip_first_load && it == 0))
                        tma_load_2d(x_base + stage * x_bytes, x_map, full_bar + 8 * stage, kb * BK, x_row);
                    filled |= 1u << stage;
                    fill_phase = (fill_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // drain: wait (bounded) for the copies this thread issued
                for (int s = 0; s < C::STAGES; ++s) {
                    if (!(filled >> s & 1u)) continue;
                    const uint64_t t0 = global_timer();
                    while (!mbar_try_wait(full_bar + 8 * s, (fill_phase >> s) & 1u) &&
                           global_timer() - t0 < WAIT_LIMIT_NS / 4) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_bf16(BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
                int mb, nb, sp, kb0, kb1;
                ts.get(t, mb, nb, sp, kb0, kb1);
                if (!mbar_wait(tempty_bar + 8 * acc, acc_phase ^ 1u, abort_flag, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(full_bar + 8 * stage, phase, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = sw128_desc(sA + stage * C::A_BYTES);
                    const uint64_t db = sw128_desc(sB + stage * C::B_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)   // +32 bytes along K per step (encoded >> 4)
                        umma_bf16(d_tmem, da + 2 * k, db + 2 * k, IDESC, (kb > kb0 || k > 0) ? 1u : 0u);
                    umma_commit(empty_bar + 8 * stage);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(tfull_bar + 8 * acc);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // on the abort path the last products may still be running (on the normal
            // path the epilogue has waited for every tile's products)
            if (!ok) mma_drain(drain_bar);
        }
    } else {
        // ------------------------------------------------ epilogue warps 2..5
        const int quarter = warp & 3;                    // TMEM lanes [32*quarter, 32*quarter + 32)
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        int acc = 0;
        uint32_t acc_phase = 0;
        pdl_wait();
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
            int mb, nb, sp, kb0, kb1;
            ts.get(t, mb, nb, sp, kb0, kb1);
            if (!mbar_wait(tfull_bar + 8 * acc, acc_phase, abort_flag, err)) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + lane_addr + (uint32_t)(acc * BN);
            const int row = mb * BM + quarter * 32 + lane;   // row of operand A
            if constexpr (MODE == EPI_SWIGLU) {
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    float g[32], u[32];
                    tmem_ld32(tacc + c * 32, g);
                    tmem_ld32(tacc + 128 + c * 32, u);
                    if (row < ep.M) epi_swiglu32<bf16>(ep, row, nb * 128 + c * 32, g, u);
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    float v[32];
                    tmem_ld32(tacc + c * 32, v);
                    const int n0 = nb * BN + c * 32;
                    if (row < ep.M && n0 < ep.N) {
                        if constexpr (MODE == EPI_F32) epi_f32_32(ep, row, n0, v);
                        else if constexpr (MODE == EPI_RESID) epi_resid32(ep, row, n0, v);
                        else epi_qkv32<bf16>(ep, row, n0, v);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(tempty_bar + 8 * acc);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS)
                     : "memory");
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 2-D K-major bf16 map: dims (K, rows), box (64, box_rows), 128-byte swizzle,
// out-of-range rows read as zero.
int make_map(CUtensorMap* map, const void* ptr, int rows, int K, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return LLAMA_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? LLAMA_OK : LLAMA_ERR_CUDA;
}

// SM count of the current device (looked up once per device)
int num_sms() {
    static std::atomic<int> cached[LLAMA_MAX_DEVICES];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= LLAMA_MAX_DEVICES) return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

template <int BN, int MODE>
int ensure_attr() {
    static PerDeviceOnce once;
    return once_per_device(once, []() -> int {
        LLAMA_CUDA_TRY(cudaFuncSetAttribute(gemm_tc_kernel<BN, MODE>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<BN>::SMEM));
        return (int)LLAMA_OK;
    });
}

template <int BN, int MODE>
int run(const CUtensorMap& ma, const CUtensorMap& mb, const TileSched& ts, const EpiArgs& a, int* err,
        cudaStream_t st) {
    using C = Cfg<BN>;
    int rc = ensure_attr<BN, MODE>();
    if (rc) return rc;
    const int tiles = ts.m_blocks * ts.n_blocks * ts.splits;
    const int grid = tiles < num_sms() ? tiles : num_sms();
    launch_pdl(gemm_tc_kernel<BN, MODE>, dim3(grid), dim3(NTHREADS), C::SMEM, st, ma, mb, ts, a, err);
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}

}  // namespace

int gemm_tc_prepare() {
    if (!encode_fn()) return LLAMA_ERR_CUDA;
    num_sms();
    int rc;
    if ((rc = ensure_attr<256, EPI_F32>())) return rc;
    if ((rc = ensure_attr<256, EPI_RESID>())) return rc;
    if ((rc = ensure_attr<256, EPI_SWIGLU>())) return rc;
    return ensure_attr<256, EPI_QKV>();
}

int gemm_tc_pick_splits(int rowsA, int K) {
    const int m_blocks = (rowsA + BM - 1) / BM;
    const int kb = K / BK;
    const int sms = num_sms();
    int best = 1;
    double best_eff = 0.0;
    for (int s = 1; s <= 16 && s <= kb / 2; ++s) {
        const int per = (kb + s - 1) / s;
        if ((s - 1) * per >= kb) continue;        // the last split would own no k-block
        const int tiles = m_blocks * s;
        const int waves = (tiles + sms - 1) / sms;
        double eff = (double)tiles / (double)(waves * sms);
        if (tiles < sms) eff *= 0.5;              // leaves SMs idle
        eff -= 0.004 * s;                         // partial-sum traffic and reduction work
        if (eff > best_eff + 1e-9) {
            best_eff = eff;
            best = s;
        }
    }
    return best;
}

int launch_gemm_tc(const TcGemm& g, int mode, const EpiArgs& a, int* err, cudaStream_t st) {
    if (g.K % BK != 0 || g.K <= 0 || g.rowsA <= 0 || g.rowsB <= 0) return LLAMA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(g.A) | reinterpret_cast<uintptr_t>(g.B)) & 15u) return LLAMA_ERR_INVALID_ARG;
    CUtensorMap ma, mb;
    TileSched ts;
    ts.skip_first_load = g.test_skip_load;
    ts.kb_total = g.K / BK;
    ts.group = 16;
    if (g.swap) return LLAMA_ERR_INVALID_ARG;   // decode projections run in decode_step.cu
    constexpr int BN = 256;
    ts.m_blocks = (g.rowsA + BM - 1) / BM;
    ts.n_blocks = (g.rowsB + BN - 1) / BN;
    ts.splits = 1;
    if (mode == EPI_SWIGLU && g.rowsB % 256 != 0) return LLAMA_ERR_INVALID_ARG;
    if ((mode == EPI_RESID || mode == EPI_QKV) && g.rowsB % 32 != 0) return LLAMA_ERR_INVALID_ARG;
    int rc = make_map(&ma, g.A, g.rowsA, g.K, BM);
    if (rc) return rc;
    rc = make_map(&mb, g.B, g.rowsB, g.K, BN);
    if (rc) return rc;
    switch (mode) {
        case EPI_F32: return run<BN, EPI_F32>(ma, mb, ts, a, err, st);
        case EPI_RESID: return run<BN, EPI_RESID>(ma, mb, ts, a, err, st);
        case EPI_SWIGLU: return run<BN, EPI_SWIGLU>(ma, mb, ts, a, err, st);
        case EPI_QKV: return run<BN, EPI_QKV>(ma, mb, ts, a, err, st);
        default: return LLAMA_ERR_INVALID_ARG;
    }
}

int tc_make_map_2d(CUtensorMap* map, const void* ptr, int rows, int K, int box_rows) {
    return make_map(map, ptr, rows, K, box_rows);
}

int tc_num_sms() { return num_sms(); }
