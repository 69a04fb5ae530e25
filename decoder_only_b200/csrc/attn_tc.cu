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
// -- a pair of adjacent 128-query tiles a, b of one (head, sequence), which
// share every key / value tile they read -- that it claims from a global
// counter; the rings and barriers run on over item boundaries, so the next
// item's Q, K and first scores load and compute while the current item's
// output is written.  Sharing each key / value tile between two query tiles
// halves the bytes streamed from L2 per product: with one query tile per
// CTA the TMA delivery of K and V (about 23 B per clock per SM with the
// products and the softmax running) bounded the kernel.
//   warp 0      TMA: lane 0 claims the items, loads each item's Q tiles
//               (once the previous item's last Q K^T products are done),
//               then its K_j tiles (three-stage ring); lane 1 the V_j tiles
//               (two stages).  3-D tensor maps (hd, position, head) make
//               rows >= S read as 0.
//   warp 1      TMEM allocator + MMA issuer, an event loop over x in {a, b}:
//                 S_x = Q_x K_j^T    (M 128, N 128, K hd)  -> TMEM S_x
//                 O_x += P_x V_j     (M 128, N hd, K 128)  -> TMEM O_x
//               P_x is the A operand read from tensor memory (written over
//               S_x by the softmax), V the MN-major B operand (hd
//               contiguous), so the cache layout [position][hd] is used as
//               is.  S_x(j + 1) is computed once P_x(j) V_j has completed
//               (it overwrites the P_x it read); meanwhile the other tile's
//               products run, so one tile's softmax overlaps the other's
//               MMAs.
//   warps 2..5  softmax of tile a, warps 6..9 of tile b, one query row per
//               thread: the row's 128 scores into registers (one TMEM read),
//               row max (pass 1), then p = 2^(s log2e / sqrt(hd) - m) rounded
//               to bf16 into the row's TMEM lane and the row sum in fp32
//               (pass 2).  The running maximum m (log2 units) moves only when
//               a tile's maximum exceeds it by more than 8: p stays <= 2^8,
//               exact in fp32 and bf16's range, and the output in TMEM is
//               rescaled by 2^(m_old - m_new) (TMEM load, scale, store) only
//               then -- a few times per row -- instead of folding every
//               tile's product into registers.  After an item's last tile:
//               O_x / (row sum), bf16, to global; the next item's first
//               P_x V product waits for that read.
// All mbarrier waits are bounded (see tcgen05.cuh).
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace {

using namespace tc;

constexpr int BQ = 128;         // queries per tile
constexpr int BKV = 128;        // keys per tile
constexpr int NTHREADS = 320;   // warp 0 TMA, warp 1 MMA, warps 2..5 softmax of tile a, 6..9 of tile b
constexpr float RESCALE_LOG2 = 8.f;   // move the running maximum only by more than this (log2 units)

// 2^x by the special-function unit's approximation (one instruction;
// relative error far below bf16's 2^-9; 2^-inf = 0 for masked scores)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

constexpr int NSK = 3;          // stages of the key ring
constexpr int NSV = 2;          // stages of the value ring

// mbarrier byte offsets in the barrier region (derived from the ring depths,
// so that changing a depth cannot make two barriers share a word)
constexpr int B_QFULL = 0, B_QEMPTY = 8, B_KFULL = 16;
constexpr int B_KEMPTY = B_KFULL + 8 * NSK, B_VFULL = B_KEMPTY + 8 * NSK;
constexpr int B_VEMPTY = B_VFULL + 8 * NSV, B_SFULL = B_VEMPTY + 8 * NSV;
constexpr int B_PFULL = B_SFULL + 16, B_PVDONE = B_PFULL + 16, B_OLAST = B_PVDONE + 16;
constexpr int B_OFREE = B_OLAST + 16, B_IFULL = B_OFREE + 16, B_IEMPTY = B_IFULL + 16;
constexpr int B_WORDS = 256;    // tensor-memory slot, abort flag, item ring after the barriers
static_assert(B_IEMPTY + 16 <= B_WORDS, "mbarrier region");

template <int HD>
struct ACfg {
    static constexpr int REG = 128 * 128;                    // one [128 rows][64 bf16] swizzled region, bytes
    static constexpr int NREG = HD / 64;                     // regions per Q / K / V tile
    static constexpr int TILE = NREG * REG;                  // Q, K or V tile bytes
    static constexpr int OFF_Q = 0;                          // [2]: tiles a, b
    static constexpr int OFF_K = OFF_Q + 2 * TILE;           // [NSK]
    static constexpr int OFF_V = OFF_K + NSK * TILE;         // [NSV]
    static constexpr int OFF_BAR = OFF_V + NSV * TILE;
    static constexpr int SMEM = OFF_BAR + 512 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;               // S / P of tiles a, b at 0, 128; O at 256, 384
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

// Non-blocking probe of an mbarrier phase (for the MMA issuer's event loop).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// A x B with A (M x K, bf16) read from tensor memory: row m in lane m, K along
// the columns, two values per 32-bit column; B from shared memory.
__device__ __forceinline__ void umma_bf16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}

// 32 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
        "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

template <int HD>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, bf16* __restrict__ out, int H, int S,
                           int Hkv, int B, float scale_log2, const int* __restrict__ pages, int pps, int hblk,
                           int* sched, int* err) {
    using C = ACfg<HD>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t sQ = base + C::OFF_Q, sK = base + C::OFF_K, sV = base + C::OFF_V;
    const uint32_t bars = base + C::OFF_BAR;
    const uint32_t q_full = bars + B_QFULL;
    const uint32_t q_empty = bars + B_QEMPTY;    // one phase per work item: its last Q K^T products done
    const uint32_t k_full = bars + B_KFULL;      // [NSK]
    const uint32_t k_empty = bars + B_KEMPTY;    // [NSK] every Q K_j^T of the key tile done
    const uint32_t v_full = bars + B_VFULL;      // [NSV]
    const uint32_t v_empty = bars + B_VEMPTY;    // [NSV] every P V_j of the value tile done
    const uint32_t s_full = bars + B_SFULL;      // [2] per query tile x: S_x(n) in TMEM
    const uint32_t p_full = bars + B_PFULL;      // [2] per x: P_x(n) in TMEM (and O_x rescaled); 128 arrivals
    const uint32_t pv_done = bars + B_PVDONE;    // [2] per x: P_x(n) V done -- S_x / P_x free, O_x current
    const uint32_t o_last = bars + B_OLAST;      // [2] per x: the item's last P_x V done
    const uint32_t o_free = bars + B_OFREE;      // [2] per x: O_x read out of TMEM; 128 arrivals
    const uint32_t item_full = bars + B_IFULL;   // [2] a work item's index published in item_ring
    const uint32_t item_empty = bars + B_IEMPTY; // [2] read by the ten consumers (V lane, MMA, 8 softmax warps)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_BAR + B_WORDS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* item_ring = reinterpret_cast<volatile int*>(tmem_slot + 2);   // [2]

    // Work items: a pair of adjacent 128-query tiles a = 2p, b = 2p + 1 of one
    // (head, sequence), which share every key / value tile they read (b reads
    // one more).  Items come in blocks of hblk heads, longest (most key tiles)
    // first within a block, so the items running at one time share the key
    // and value tiles of a few heads in L2.  Each CTA starts with item
    // blockIdx.x and then claims the next unclaimed one from a global counter
    // (sched[0]) whenever it is ready for another; lane 0 of warp 0 claims and
    // publishes them to the other roles through a two-entry ring.  All rings
    // and barriers run on across items.
    const int n_qt = (S + BQ - 1) / BQ;
    const int n_qp = (n_qt + 1) / 2;
    const int total = n_qp * H * B;
    const int G = (int)gridDim.x;
    auto item = [&](int it, int& pr, int& h, int& b) {
        const int per = hblk * n_qp;
        const int k = it / per;
        const int r = it - k * per;
        const int gg = min(hblk, H * B - k * hblk);
        pr = n_qp - 1 - r / gg;
        const int hb = k * hblk + r % gg;
        h = hb % H;
        b = hb / H;
    };
    // consumer side of the item ring: the index of this role's ni-th item
    auto next_item = [&](int ni, bool& ok) -> int {
        const int slot = ni & 1;
        ok = mbar_wait(item_full + 8 * slot, (uint32_t)((ni >> 1) & 1), abort_flag, err);
        return ok ? item_ring[slot] : total;
    };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < NSK; ++i) {
            mbar_init(k_full + 8 * i, 1);
            mbar_init(k_empty + 8 * i, 1);
        }
        for (int i = 0; i < NSV; ++i) {
            mbar_init(v_full + 8 * i, 1);
            mbar_init(v_empty + 8 * i, 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(s_full + 8 * x, 1);
            mbar_init(p_full + 8 * x, 128);
            mbar_init(pv_done + 8 * x, 1);
            mbar_init(o_last + 8 * x, 1);
            mbar_init(o_free + 8 * x, 128);
            mbar_init(item_full + 8 * x, 1);
            mbar_init(item_empty + 8 * x, 10);
        }
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
            // lane 0: claims and publishes the items; each item's Q tiles (once the
            // previous item's last Q K^T products are done), then its K_j; lane 1: the V_j
            const bool is_k = (lane == 0);
            const int ns = is_k ? NSK : NSV;
            const uint32_t full = is_k ? k_full : v_full, empty = is_k ? k_empty : v_empty;
            const uint32_t dst = is_k ? sK : sV;
            const CUtensorMap* map = is_k ? &tmK : &tmV;
            bool ok = true;
            int kt = 0, ni = 0, q_loads = 0;
            int it = blockIdx.x;
            for (;; ++ni) {
                if (is_k) {
                    // publish item ni (after all ten consumers have read item ni - 2 from its slot)
                    const int slot = ni & 1;
                    if (ni >= 2 && !mbar_wait(item_empty + 8 * slot, (uint32_t)(((ni >> 1) - 1) & 1), abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    item_ring[slot] = it;
                    mbar_arrive(item_full + 8 * slot);
                } else {
                    it = next_item(ni, ok);
                    if (!ok) break;
                    mbar_arrive(item_empty + 8 * (ni & 1));
                }
                if (it >= total) break;
                int pr, h, b;
                item(it, pr, h, b);
                const bool has_b = 2 * pr + 1 < n_qt;
                const int nk = has_b ? 2 * pr + 2 : 2 * pr + 1;     // key tiles of the pair
                const int kv_head = b * Hkv + h / (H / Hkv);      // grouped keys and values
                if (is_k) {
                    if (ni > 0 && !mbar_wait(q_empty, (uint32_t)((ni - 1) & 1), abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(q_full, (has_b ? 2 : 1) * C::TILE);
                    for (int r = 0; r < C::NREG; ++r) {
                        tma_load_3d(sQ + r * C::REG, &tmQ, q_full, 64 * r, 2 * pr * BQ, b * H + h);
                        if (has_b) tma_load_3d(sQ + C::TILE + r * C::REG, &tmQ, q_full, 64 * r, (2 * pr + 1) * BQ, b * H + h);
                    }
                    ++q_loads;
                }
                for (int j = 0; j < nk; ++j, ++kt) {
                    const int st = kt % ns;
                    if (!mbar_wait(empty + 8 * st, ((kt / ns) & 1) ^ 1u, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(full + 8 * st, C::TILE);
                    for (int r = 0; r < C::NREG; ++r)
                        // paged cache: key tile j is page pages[b][j] (KV_PAGE == BKV positions)
                        tma_load_3d(dst + st * C::TILE + r * C::REG, map, full + 8 * st, 64 * r, pages ? 0 : j * BKV,
                                    pages ? __ldg(pages + b * pps + j) * Hkv + (kv_head - b * Hkv) : kv_head);
                }
                if (!ok) break;
                if (is_k) it = G + atomicAdd(sched, 1);   // claim the next item
            }
            if (!ok) {
                // drain (bounded) the copies this thread issued
                const uint64_t t0 = global_timer();
                while (is_k && q_loads > 0 && !mbar_try_wait(q_full, (uint32_t)((q_loads - 1) & 1)) &&
                       global_timer() - t0 < WAIT_LIMIT_NS / 4) {
                }
                for (int t = kt > ns ? kt - ns : 0; t < kt; ++t) {
                    const uint32_t par = (t / ns) & 1;
                    while (!mbar_try_wait(full + 8 * (t % ns), par) && global_timer() - t0 < WAIT_LIMIT_NS / 2) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        // An event loop over the two query tiles x: S_x(j) = Q_x K_j^T once K_j has
        // landed and the previous P_x V product has completed (S_x(j) overwrites
        // the P_x it read); O_x += P_x(j) V_j once the softmax has written P_x(j)
        // and V_j has landed.  One tile's softmax overlaps the other tile's products.
        if (lane == 0) {
            constexpr uint32_t IDESC_QK = idesc_bf16(BKV);                 // K-major A and B
            constexpr uint32_t IDESC_PV = idesc_bf16(HD) | (1u << 16);      // B (V) MN-major
            bool ok = true;
            int kv0 = 0;                                // key / value tiles of earlier items
            int sc[2] = {0, 0}, pc[2] = {0, 0};         // S_x / P_x V products issued so far (all items)
            int nix[2] = {0, 0};                        // items in which tile x took part
            for (int ni = 0; ok; ++ni) {
                const int it = next_item(ni, ok);
                if (!ok) break;
                mbar_arrive(item_empty + 8 * (ni & 1));
                if (it >= total) break;
                int pr, h, b;
                item(it, pr, h, b);
                const bool has_b = 2 * pr + 1 < n_qt;
                const int nkx[2] = {2 * pr + 1, has_b ? 2 * pr + 2 : 0};
                const int nk = has_b ? nkx[1] : nkx[0];
                ok = mbar_wait(q_full, (uint32_t)(ni & 1), abort_flag, err);
                tc_fence_after();
                int js[2] = {0, 0}, jp[2] = {0, 0};     // this item's next S_x / P_x V tile
                int krel = 0, vrel = 0;
                bool q_rel = false;
                uint64_t t_last = global_timer();
                while (ok && (krel < nk || vrel < nk || !q_rel)) {
                    bool prog = false;
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        // O_x += P_x(j) V_j
                        const int j = jp[x];
                        if (j < js[x] && mbar_test(p_full + 8 * x, (uint32_t)(pc[x] & 1)) &&
                            mbar_test(v_full + 8 * ((kv0 + j) % NSV), (uint32_t)(((kv0 + j) / NSV) & 1)) &&
                            (j > 0 || nix[x] == 0 || mbar_test(o_free + 8 * x, (uint32_t)((nix[x] - 1) & 1)))) {
                            tc_fence_after();
                            const uint32_t d_o = tmem + 256u + 128u * x;
                            const uint32_t p_t = tmem + 128u * x;     // P_x over S_x's first 64 columns
                            const uint32_t v_t = sV + ((kv0 + j) % NSV) * C::TILE;
#pragma unroll
                            for (int kk = 0; kk < BKV / 16; ++kk) {
                                // A = P from TMEM (16 keys = 8 columns); B = V (MN-major): 16 keys = 2 groups of 8 rows
                                uint64_t vd = sw128_desc(v_t + kk * 2048);
                                vd = (vd & ~(((uint64_t)0x3FFF) << 16)) | ((uint64_t)(C::REG >> 4) << 16);   // LBO: next 64 hd
                                umma_bf16_tmem_a(d_o, p_t + 8u * kk, vd, IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
                            }
                            umma_commit(pv_done + 8 * x);
                            if (j == nkx[x] - 1) umma_commit(o_last + 8 * x);
                            ++pc[x];
                            jp[x] = j + 1;
                            prog = true;
                        }
                    }
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        // S_x(j) = Q_x K_j^T
                        const int j = js[x];
                        if (j < nkx[x] && jp[x] == j &&
                            mbar_test(k_full + 8 * ((kv0 + j) % NSK), (uint32_t)(((kv0 + j) / NSK) & 1)) &&
                            (sc[x] == 0 || mbar_test(pv_done + 8 * x, (uint32_t)((sc[x] - 1) & 1)))) {
                            tc_fence_after();
                            const uint32_t d_s = tmem + 128u * x;
                            const uint32_t q_t = sQ + x * C::TILE, k_t = sK + ((kv0 + j) % NSK) * C::TILE;
#pragma unroll
                            for (int kk = 0; kk < HD / 16; ++kk) {
                                const uint32_t off = (kk >> 2) * C::REG + (kk & 3) * 32;
                                umma_bf16(d_s, sw128_desc(q_t + off), sw128_desc(k_t + off), IDESC_QK,
                                          kk > 0 ? 1u : 0u);
                            }
                            umma_commit(s_full + 8 * x);
                            ++sc[x];
                            js[x] = j + 1;
                            prog = true;
                        }
                    }
                    // release key / value tiles once every product that reads them is issued,
                    // and the Q tiles once both tiles' last Q K^T is
                    while (krel < nk && (krel >= nkx[0] || js[0] > krel) && (krel >= nkx[1] || js[1] > krel)) {
                        umma_commit(k_empty + 8 * ((kv0 + krel) % NSK));
                        ++krel;
                        prog = true;
                    }
                    while (vrel < nk && (vrel >= nkx[0] || jp[0] > vrel) && (vrel >= nkx[1] || jp[1] > vrel)) {
                        umma_commit(v_empty + 8 * ((kv0 + vrel) % NSV));
                        ++vrel;
                        prog = true;
                    }
                    if (!q_rel && js[0] == nkx[0] && js[1] == nkx[1]) {
                        umma_commit(q_empty);
                        q_rel = true;
                        prog = true;
                    }
                    if (prog) {
                        t_last = global_timer();
                        continue;
                    }
                    if (*abort_flag) {
                        ok = false;
                        break;
                    }
                    if (global_timer() - t_last > WAIT_LIMIT_NS) {
                        *abort_flag = 1;
                        atomicOr(err, LLAMA_DEVERR_TIMEOUT);
                        ok = false;
                        break;
                    }
                }
                kv0 += nk;
                nix[0] += 1;
                if (has_b) nix[1] += 1;
            }
        }
    } else {
        // ---------------------------------------------------------- softmax + output (warps 2..9)
        const int x = (warp - 2) >> 2;                   // query tile a (0) or b (1)
        const int quarter = warp & 3;
        const int t_row = quarter * 32 + lane;           // query row within the tile
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const uint32_t o_addr = tmem + lane_addr + 256u + 128u * x;
        const uint32_t s_addr = tmem + lane_addr + 128u * x;
        bool ok = true;
        int sc = 0, nix = 0;                             // S_x tiles and items of tile x so far
        for (int ni = 0; ok; ++ni) {
            bool got;
            const int it = next_item(ni, got);
            if (!__all_sync(0xffffffffu, got)) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(item_empty + 8 * (ni & 1));
            if (it >= total) break;
            int pr, h, b;
            item(it, pr, h, b);
            const int qt = 2 * pr + x;
            if (qt >= n_qt) continue;                    // the pair's second tile lies past S
            const int n_kv = qt + 1;
            const int q = qt * BQ + t_row;
            float m = -INFINITY, l = 0.f;                // running maximum (log2 units) and row sum
            for (int j = 0; j < n_kv; ++j, ++sc) {
                // warp-uniform decision: the TMEM loads below are warp-collective
                if (!__all_sync(0xffffffffu, mbar_wait(s_full + 8 * x, (uint32_t)(sc & 1), abort_flag, err))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
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
                // pass 2: probabilities (bf16 pairs, key 2c in the low half of
                // column c) into this row's TMEM lane over the first 64 columns
                // of S_x (read out above); the row sum adds the fp32 values in
                // four independent partial sums
                float rs4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float p0 = ex2_approx(fmaf(sv[64 * half + 2 * i], scale_log2, -m));
                        const float p1 = ex2_approx(fmaf(sv[64 * half + 2 * i + 1], scale_log2, -m));
                        pk[i] = pack_bf16x2(p0, p1);
                        rs4[i & 3] += p0 + p1;
                    }
                    tmem_st32u(s_addr + 32 * half, pk);
                }
                const float rs = (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
                tmem_st_wait();
                // a warp with a moved maximum rescales its 32 rows of O_x: the
                // previous P_x V product has completed (S_x(j) was issued after it)
                if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                    for (int c = 0; c < HD / 32; ++c) {
                        float ov[32];
                        tmem_ld32(o_addr + c * 32, ov);
#pragma unroll
                        for (int i = 0; i < 32; ++i) ov[i] *= corr;
                        tmem_st32(o_addr + c * 32, ov);
                    }
                    tmem_st_wait();
                }
                l = l * corr + rs;
                tc_fence_before();
                mbar_arrive(p_full + 8 * x);
            }
            // the tile's last product: O_x / l, bf16, to global; then O_x is free for the next item
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_last + 8 * x, (uint32_t)(nix & 1), abort_flag, err));
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
            mbar_arrive(o_free + 8 * x);
            ++nix;
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
    if (threadIdx.x == 0) {
        // this CTA claims no more items; the last CTA to finish zeroes the
        // counters for the next launch
        __threadfence();
        if (atomicAdd(sched + 1, 1) == G - 1) {
            atomicExch(sched, 0);
            atomicExch(sched + 1, 0);
        }
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
                                int hd, int kv_stride, int* err, int* sched, cudaStream_t st, const int* pages, int pps,
                                int n_pages) {
    if (B <= 0 || S <= 0) return LLAMA_OK;
    if (!sched) return LLAMA_ERR_INVALID_ARG;
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
    const int items = (((S + BQ - 1) / BQ + 1) / 2) * H * B;
    const int n_sm = tc_num_sms();
    dim3 grid(items < n_sm ? items : n_sm);
    // heads per block of work items: the key and value bytes of a block's
    // heads (all positions) about 32 MB, so two blocks in flight stay well
    // inside L2; at least 8 heads, for the balance of the CTAs' loads
    const double kv_head_bytes = 4.0 * S * hd / (H / Hkv);
    int hblk = (int)(32.0 * (1 << 20) / kv_head_bytes);
    hblk = std::max(8, std::min(hblk, H * B));
    if (hd == 128) {
        if ((rc = attn_attr<128>())) return rc;
        launch_pdl(attn_prefill_tc_kernel<128>, grid, dim3(NTHREADS), ACfg<128>::SMEM, st, mq, mk, mv, (bf16*)o, H, S,
                   Hkv, B, scale_log2, pages, pps, hblk, sched, err);
    } else {
        if ((rc = attn_attr<64>())) return rc;
        launch_pdl(attn_prefill_tc_kernel<64>, grid, dim3(NTHREADS), ACfg<64>::SMEM, st, mq, mk, mv, (bf16*)o, H, S,
                   Hkv, B, scale_log2, pages, pps, hblk, sched, err);
    }
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}
