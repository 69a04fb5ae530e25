// The greedy decode step of a bf16 model as one persistent kernel.
//
// One decode step ([PFD] "The one formula" applied to the B newest tokens,
// keys and values of all earlier positions read from the cache ([NAR] "GQA
// Was Not an Original LLaMA Feature")) is a chain of small, HBM-bound
// phases:
//   embed (+ the first norm's inputs)
//   per layer:  QKV projection (+RoPE, append K and V at each sequence's position)
//               attention over the cache
//               O projection (+residual, + the FFN norm's inputs)
//               gate/up projection (+SwiGLU)
//               down projection (+residual, + the next norm's inputs)
//   head projection (fp32 logits), greedy argmax, positions + 1.
// Launched one kernel per phase, fixed costs dominate (launch, set-up,
// pipeline fill, tails).  Here one cooperative launch of one CTA per SM runs
// all phases.  Phases are ordered by completion counts, not grid barriers:
// every unit of work that a later phase reads (a finished 128-row block of a
// projection, a finished attention pair) adds one to a count per (layer,
// kind), and a consumer waits only for the count it depends on.  The
// weights -- which depend on no phase -- stream continuously: the TMA
// producer keeps its ring of weight tiles full across phase boundaries, and
// only the activation tile of each stage waits for its phase's input.
//
// Work split of a projection: its (128-row block, 64-wide k-block)
// iterations, block-major, are cut into gridDim.x equal contiguous ranges
// (stream-K), so every CTA streams the same number of weight bytes and
// finishes at most a few accumulators per phase.  A block touched by one
// range is finished directly from the accumulator; otherwise each range
// leaves a partial sum and the last range to arrive adds them in range
// order (deterministic) and finishes the block.
//
// RMSNorm ([PFD] "RMSNorm: LayerNorm minus the mean") enters a projection as
// W (g * x / rms(x)).  1/rms(x) is one scalar per token, so it commutes with
// W: the code that finishes a 128-feature block of the trunk x writes
// bf16(g * x) and the block's sum of squares; the projection consuming the
// norm multiplies its fp32 result by rsqrt(sum of the block sums / d + eps),
// the block sums added in a fixed order.  No phase waits on a separate
// normalisation pass over the whole trunk.  (The bias variant's norm shift
// beta enters the same way: W beta is folded into that projection's bias.)
//
// Warp roles (256 threads):
//   warps 0-3  projection epilogues, attention, greedy choice
//   warp 4     TMA producer, all projections of the step in order
//   warp 5     TMEM owner and tcgen05.mma issuer (swap-AB: 128 weight rows on
//              the TMEM lanes, the B <= 32 tokens as N = 16 or 32 columns)
//   warps 6-7  attention
// Every wait is bounded (2 s): a CTA that gives up records
// LLAMA_DEVERR_TIMEOUT and leaves; the others then give up at their own next
// wait.  Named barriers among the 128 epilogue threads follow a collective
// OR of each thread's wait result, so they leave together.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace {

using namespace tc;

constexpr int BM = 128;      // weight rows per tile (TMEM lanes)
constexpr int BK = 64;       // K per stage (one 128-byte swizzle row)
constexpr int NT = 256;      // warps 0-3 epilogue, 4 TMA producer, 5 MMA, 6-7 attention
constexpr int NAW = STEP_ATTN_WARPS;   // attention warps per CTA: the four epilogue warps and warps 6, 7
static_assert(NAW == 6, "warp roles");
static_assert(KV_PAGE % 16 == 0, "an attention chunk stays inside one page");
constexpr int ACH = 16;      // keys per attention chunk (one bulk copy of K rows, one of V rows)
constexpr int AMX = 2048;    // logits per greedy-choice item
constexpr int SSQ_BLOCKS = 64;   // 128-feature blocks of one norm's sums of squares (d <= 8192)

enum PhaseType { PH_EMBED = 0, PH_QKV = 1, PH_ATTN = 2, PH_O = 3, PH_GU = 4, PH_DOWN = 5, PH_HEAD = 6, PH_ARGMAX = 7 };

template <int BN, int HD>
struct SCfg {
    static constexpr int STAGES = (BN == 16) ? 5 : 4;
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    // attention: per attention warp two chunk buffers (K rows, V rows, and
    // the query of a pair whose first chunk it is); the transpose buffer of
    // the projection epilogues shares the region
    static constexpr int ATT_Q = 2 * ACH * HD * 2;                        // offset of the query
    static constexpr int ATT_BUF = ATT_Q + HD * 2;
    static constexpr int OFF_ATT = OFF_B + STAGES * B_BYTES;             // [NAW warps][2][ATT_BUF]
    static constexpr int OFF_X = OFF_ATT;                                 // [32][XLD] floats
    static constexpr int XLD = BM + 1;
    static constexpr int ATT_BYTES = NAW * 2 * ATT_BUF > 32 * XLD * 4 ? NAW * 2 * ATT_BUF : 32 * XLD * 4;
    static constexpr int OFF_SML = OFF_ATT + ATT_BYTES;                   // 1/rms [32], reduction scratch
    static constexpr int OFF_BAR = OFF_SML + 1024;                       // mbarriers, then misc words
    static constexpr int OFF_MISC = OFF_BAR + 8 * (2 * STAGES + 4 + 2 * NAW);
    static constexpr int SMEM = OFF_BAR + 512 + 1024;
    static_assert(OFF_MISC + 16 <= OFF_BAR + 512, "mbarrier region");
    static constexpr uint32_t TMEM_COLS = (2 * BN < 32) ? 32 : 2 * BN;
};

__device__ __forceinline__ int phase_count(const StepArgs& a) { return 3 + 5 * a.L; }

__device__ __forceinline__ int phase_type(const StepArgs& a, int p, int& layer) {
    if (p == 0) {
        layer = 0;
        return PH_EMBED;
    }
    const int q = p - 1;
    if (q < 5 * a.L) {
        layer = q / 5;
        return PH_QKV + q % 5;
    }
    layer = a.L;
    return q == 5 * a.L ? PH_HEAD : PH_ARGMAX;
}

// One projection: weight map, activation map, output rows, K, epilogue and
// its kind (index of its partial / counter region)
struct GemmPh {
    int map_a, map_b, rowsA, K, mode, kind;
};

__device__ __forceinline__ bool gemm_of(const StepArgs& a, int type, int l, GemmPh& g) {
    const int L = a.L;
    switch (type) {
        case PH_QKV: g = GemmPh{4 * l + 0, 4 * L + 1, a.d + 2 * a.Hkv * a.hd, a.d, EPI_QKV, 0}; return true;
        case PH_O: g = GemmPh{4 * l + 1, 4 * L + 2, a.d, a.d, EPI_RESID, 1}; return true;
        case PH_GU: g = GemmPh{4 * l + 2, 4 * L + 4, 2 * a.h, a.d, EPI_SWIGLU, 2}; return true;
        case PH_DOWN: g = GemmPh{4 * l + 3, 4 * L + 3, a.d, a.h, EPI_RESID, 3}; return true;
        case PH_HEAD: g = GemmPh{4 * L, 4 * L + 1, a.V, a.d, EPI_F32, 4}; return true;
        default: return false;
    }
}

// This CTA's stream-K range [s, e) of a projection's T = mblk * kbt
// iterations (iteration i: block i / kbt, k-block i % kbt), cut into
// G = min(gridDim.x, T) equal ranges so that none is empty; CTAs from G on
// have no work in this projection.
struct Work {
    GemmPh g;
    int mblk, kbt, s, e, G;
    long long T;
};

__device__ __forceinline__ bool work_of(const StepArgs& a, int type, int l, Work& w) {
    if (!gemm_of(a, type, l, w.g)) return false;
    w.mblk = w.g.rowsA / BM;
    w.kbt = w.g.K / BK;
    w.T = (long long)w.mblk * w.kbt;
    w.G = (int)min((long long)gridDim.x, w.T);
    const int c = blockIdx.x;
    w.s = c < w.G ? (int)(w.T * c / w.G) : 0;
    w.e = c < w.G ? (int)(w.T * (c + 1) / w.G) : 0;
    return true;
}

// The CTA whose range holds iteration i: the largest c with c*T/G <= i
__device__ __forceinline__ int owner_of(long long i, const Work& w) { return (int)(((i + 1) * w.G - 1) / w.T); }

// Walk over this CTA's projection iterations of the whole step, in order.
struct Cursor {
    int p, i, e, kbt, mb, kb, map_a, map_b;
    const unsigned* dep;   // completion count this phase's activations wait for (nullptr: none)
    unsigned tgt;
    bool valid;
};

__device__ const unsigned* dep_of(const StepArgs& a, int type, int l, unsigned& target);

__device__ void cursor_seek(const StepArgs& a, int P, Cursor& c, int p0) {
    for (int p = p0; p < P; ++p) {
        int l;
        const int type = phase_type(a, p, l);
        Work w;
        if (!work_of(a, type, l, w) || w.s >= w.e) continue;
        c.p = p;
        c.i = w.s;
        c.e = w.e;
        c.kbt = w.kbt;
        c.mb = w.s / w.kbt;
        c.kb = w.s - c.mb * w.kbt;
        c.map_a = w.g.map_a;
        c.map_b = w.g.map_b;
        c.dep = dep_of(a, type, l, c.tgt);
        c.valid = true;
        return;
    }
    c.valid = false;
}

// Next iteration: block and k-block advance without a division
__device__ __forceinline__ void cursor_next(const StepArgs& a, int P, Cursor& c) {
    if (++c.i < c.e) {
        if (++c.kb == c.kbt) {
            c.kb = 0;
            ++c.mb;
        }
        return;
    }
    cursor_seek(a, P, c, c.p + 1);
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Non-blocking probe of an mbarrier phase
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

// Named barrier of the 128 epilogue threads
__device__ __forceinline__ void esync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// ... that also returns whether any of them passed true (all leave together)
__device__ __forceinline__ bool esync_any(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, 1, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}

// Step synchronisation words in a.bar (32-bit words; each group on a
// 128-byte line of its own).  Phases are not separated by grid barriers:
// every unit of work that produces an input of a later phase (a finished
// 128-row block of a projection, a finished attention pair) adds one to its
// completion count, and a consumer waits until the count it depends on is
// complete.
//   [0]                     epoch of the last completed step
//   [32]                    CTAs that have started the running step
//   [64]                    epoch whose embedding (and count reset) is done
//   [96]                    embedded rows of the running step
//   [128 + 32 (8 l + k)]    completion count of kind k in layer l (l = L: head)
constexpr int SY_EPOCH = 0, SY_CHECKIN = 32, SY_EMBED = 64, SY_ROWS = 96, SY_DONE = 128;
enum DoneKind { DK_QKV = 0, DK_ATTN = 1, DK_O = 2, DK_GU = 3, DK_DOWN = 4, DK_HEAD = 0 };

__device__ __forceinline__ unsigned* done_ctr(const StepArgs& a, int l, int k) {
    return a.bar + SY_DONE + 32 * (8 * l + k);
}

// Bounded wait until *p >= target (signed difference: epochs wrap)
__device__ bool wait_at_least(const unsigned* p, unsigned target, volatile int* abort_flag, int* err) {
    if ((int)(ld_acquire_u32(p) - target) >= 0) return true;
    const uint64_t t0 = global_timer();
    while (true) {
        if ((int)(ld_acquire_u32(p) - target) >= 0) return true;
        if (*abort_flag) return false;
        if (global_timer() - t0 > WAIT_LIMIT_NS) {
            *abort_flag = 1;
            atomicOr(err, LLAMA_DEVERR_TIMEOUT);
            return false;
        }
        __nanosleep(64);
    }
}

// One finished unit: a release add, so the writes of the CTA (or warp) that
// the caller's barrier ordered before it are visible to whoever acquires the
// count (release is cumulative over what happened before it)
__device__ __forceinline__ void count_done(unsigned* p) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p) : "memory");
}

// Arrival at a split counter: releases the caller's (barrier-ordered) partial
// writes and acquires the earlier arrivals', returns the previous value
__device__ __forceinline__ int arrive_acq_rel(int* p) {
    int prev;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(p) : "memory");
    return prev;
}

// The completion count (and its complete value) that phase `type` of layer
// l reads its input after; nullptr: the embedding, which every role of
// every CTA waits for before anything else.
__device__ const unsigned* dep_of(const StepArgs& a, int type, int l, unsigned& target) {
    const unsigned nd = (unsigned)(a.d / BM);
    switch (type) {
        case PH_QKV:
            target = nd;
            return l == 0 ? nullptr : done_ctr(a, l - 1, DK_DOWN);
        case PH_ATTN: target = (unsigned)((a.d + 2 * a.Hkv * a.hd) / BM); return done_ctr(a, l, DK_QKV);
        case PH_O: target = (unsigned)(a.B * a.H); return done_ctr(a, l, DK_ATTN);
        case PH_GU: target = nd; return done_ctr(a, l, DK_O);
        case PH_DOWN: target = (unsigned)(a.h / BM); return done_ctr(a, l, DK_GU);
        case PH_HEAD:
            target = nd;
            return a.L == 0 ? nullptr : done_ctr(a, a.L - 1, DK_DOWN);
        case PH_ARGMAX: target = (unsigned)(a.V / BM); return done_ctr(a, a.L, DK_HEAD);
        default: return nullptr;
    }
}

template <int BN, int HD>
struct Smem {
    uint32_t sA, sB;
    uint32_t full, empty, tfull, tempty, abar;
    uint8_t* att;        // generic pointer to the attention buffers
    float* xbuf;         // [32][XLD] transpose buffer
    float* sinv;         // [32] 1/rms of the B rows for the current projection
    float* red;          // [128] reduction scratch
    volatile int* flag;
};

// 1/rms of each of the B rows from a norm's 128-feature block sums of
// squares (added in block order by lane, then across the warp: the same
// order in every CTA), into sinv.
__device__ void load_inv(const StepArgs& a, const float* ssq, float* sinv, int tid) {
    const int warp = tid >> 5, lane = tid & 31, nblk = a.d / BM;
    for (int b = warp; b < a.B; b += 4) {
        float s = 0.f;
        for (int k = lane; k < nblk; k += 32) s += __ldcg(ssq + k * 32 + b);
        s = warp_sum(s);
        if (lane == 0) sinv[b] = rsqrtf(s / (float)a.d + a.eps);
    }
    esync();
}

// ---------------------------------------------------------------- projection epilogue
// Sum of one feature's partials, stored contiguously [slot][Mp]: every load
// is independent, issued four slots at a time, summed in slot order
// (deterministic).
template <int BN>
__device__ __forceinline__ void splitk_sum(const float* p, int slots, int M, int Mp, float (&out)[BN]) {
    constexpr int U = BN <= 16 ? 4 : 2;   // slots in flight per round (register budget)
#pragma unroll
    for (int b = 0; b < BN; ++b) out[b] = 0.f;
    if (M <= 4) {
        // one float4 per slot: eight slots per round in flight, summed in slot order
        for (int s0 = 0; s0 < slots; s0 += 8) {
            float4 w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                w[u] = (s0 + u < slots) ? __ldcg(reinterpret_cast<const float4*>(p + (size_t)(s0 + u) * Mp))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                out[0] += w[u].x;
                out[1] += w[u].y;
                out[2] += w[u].z;
                out[3] += w[u].w;
            }
        }
        return;
    }
    int s = 0;
    for (; s + U <= slots; s += U) {
        float4 w[U][BN / 4];
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int q = 0; q < BN / 4; ++q)
                w[u][q] = (4 * q < M) ? __ldcg(reinterpret_cast<const float4*>(p + (size_t)(s + u) * Mp + 4 * q))
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int q = 0; q < BN / 4; ++q) {
                out[4 * q] += w[u][q].x;
                out[4 * q + 1] += w[u][q].y;
                out[4 * q + 2] += w[u][q].z;
                out[4 * q + 3] += w[u][q].w;
            }
    }
    for (; s < slots; ++s)
#pragma unroll
        for (int q = 0; q < BN / 4; ++q)
            if (4 * q < M) {
                const float4 w = __ldcg(reinterpret_cast<const float4*>(p + (size_t)s * Mp + 4 * q));
                out[4 * q] += w.x;
                out[4 * q + 1] += w.y;
                out[4 * q + 2] += w.z;
                out[4 * q + 3] += w.w;
            }
}

// The accumulator of this CTA's range over block mb (et = TMEM lane =
// feature within the block): leave it as a partial, or finish the block.
template <int BN, int HD, int MODE>
__device__ void tile_epilogue(const StepArgs& a, const EpiArgs& ep, const Work& w, int l, int type, int mb, int et,
                              int tid, const float (&v)[32], const Smem<BN, HD>& sm) {
    constexpr bool PAIR = (MODE == EPI_SWIGLU);
    constexpr int XLD = SCfg<BN, HD>::XLD;
    const int M = a.B;
    const int Mp = (M + 3) & ~3;             // partials: [feature][slot][Mp], read back as float4
    const int ns = step_slots(w.mblk, w.G);
    auto first_of = [&](int m) { return owner_of((long long)m * w.kbt, w); };
    auto nseg_of = [&](int m) { return owner_of((long long)(m + 1) * w.kbt - 1, w) - first_of(m) + 1; };
    const int nseg = nseg_of(mb);
    const int n = mb * BM + et;
    float* part = a.partial + a.part_off[w.g.kind];
    const bool direct = (nseg == 1) && !PAIR;
    // a residual block's trunk values are final once the phase's input is
    // (the previous residual phase finished before it): read them before the
    // arrival, off the finishing range's critical path
    float tv[BN], gn = 0.f, bn = 0.f;
    if constexpr (MODE == EPI_RESID) {
#pragma unroll
        for (int b = 0; b < BN; ++b) tv[b] = (b < M) ? __ldcg(a.trunk + (size_t)b * a.d + n) : 0.f;
        // and the next norm's gain, the projection's bias (b_o / b_d) of this column
        gn = (type == PH_O ? a.gains[2 * l + 1] : a.gains[2 * (l + 1)])[n];
        bn = a.biases ? a.biases[4 * l + (type == PH_O ? 1 : 3)][n] : 0.f;
    }
    if (!direct) {
        float* dst = part + ((size_t)n * ns + ((int)blockIdx.x - first_of(mb))) * Mp;
#pragma unroll
        for (int b = 0; b < BN; b += 4)
            if (b < M) *reinterpret_cast<float4*>(dst + b) = make_float4(v[b], v[b + 1], v[b + 2], v[b + 3]);
        esync();
        int last = 0;
        if (tid == 0) {
            int* cnt = a.counters + a.cnt_off[w.g.kind] + (PAIR ? (mb >> 1) : mb);
            const int target = PAIR ? nseg_of(mb & ~1) + nseg_of(mb | 1) : nseg;
            const int prev = arrive_acq_rel(cnt);
            last = (prev == target - 1);
            if (last) *cnt = 0;   // ready for the next step; published by this CTA's later release
        }
        if (!esync_any(last)) return;
    }
    if constexpr (PAIR) {
        // hidden units 128j + et from gate feature 256j + et and up feature 256j + 128 + et
        const int j = mb >> 1;
        float gs[BN], us[BN];
        splitk_sum<BN>(part + (size_t)(256 * j + et) * ns * Mp, nseg_of(2 * j), M, Mp, gs);
        splitk_sum<BN>(part + (size_t)(256 * j + 128 + et) * ns * Mp, nseg_of(2 * j + 1), M, Mp, us);
        const float* cb = a.biases ? a.biases[4 * l + 2] : nullptr;   // folded gate / up biases
        const float bg = cb ? cb[256 * j + et] : 0.f, bu = cb ? cb[256 * j + 128 + et] : 0.f;
#pragma unroll
        for (int b = 0; b < BN; ++b)
            if (b < M) {
                const float inv = sm.sinv[b];
                a.act[(size_t)b * a.h + 128 * j + et] =
                    __float2bfloat16_rn(silu_f(gs[b] * inv + bg) * (us[b] * inv + bu));
            }
        esync();
        if (tid == 0) count_done(done_ctr(a, l, DK_GU));
    } else {
        float sum[BN];
        if (direct) {
#pragma unroll
            for (int b = 0; b < BN; ++b) sum[b] = v[b];
        } else {
            splitk_sum<BN>(part + (size_t)n * ns * Mp, nseg, M, Mp, sum);
        }
        if constexpr (MODE == EPI_F32) {
#pragma unroll
            for (int b = 0; b < BN; ++b)
                if (b < M) ep.out[(size_t)b * ep.ld_out + n] = sum[b] * sm.sinv[b];
            esync();
            if (tid == 0) count_done(done_ctr(a, a.L, DK_HEAD));
        } else if constexpr (MODE == EPI_RESID) {
            // trunk += the block's sum; then the next norm's inputs: bf16(g * x)
            // and the block's sum of squares per row
            const bool to_ffn = (type == PH_O);
            bf16* xg = to_ffn ? a.xg2 : a.xg;
#pragma unroll
            for (int b = 0; b < BN; ++b)
                if (b < M) {
                    float* o = a.trunk + (size_t)b * a.d + n;
                    const float x = tv[b] + sum[b] + bn;
                    *o = x;
                    xg[(size_t)b * a.d + n] = __float2bfloat16_rn(x * gn);
                    sm.xbuf[b * XLD + et] = x * x;
                }
            esync();
            const int warp = tid >> 5, lane = tid & 31;
            float* ssq = a.ssq + (to_ffn ? SSQ_BLOCKS * 32 : 0);
            for (int b = warp; b < M; b += 4) {
                const float* r = sm.xbuf + b * XLD;
                const float s = warp_sum((r[lane] + r[lane + 32]) + (r[lane + 64] + r[lane + 96]));
                if (lane == 0) ssq[mb * 32 + b] = s;
            }
            esync();
            if (tid == 0) count_done(done_ctr(a, l, to_ffn ? DK_O : DK_DOWN));
        } else {   // EPI_QKV: 1/rms, then RoPE and the cache append on 32-column rows
#pragma unroll
            for (int b = 0; b < BN; ++b)
                if (b < M) sm.xbuf[b * XLD + et] = sum[b] * sm.sinv[b];
            esync();
            if (tid < 4 * M) {
                const int b = tid >> 2, c = tid & 3;
                float x[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = sm.xbuf[b * XLD + c * 32 + i];
                epi_qkv32<bf16>(ep, b, mb * BM + c * 32, x);
            }
            esync();
            if (tid == 0) count_done(done_ctr(a, l, DK_QKV));
        }
    }
}

// ---------------------------------------------------------------- attention phase
// Work split: the (pair = (sequence b, head h), 16-key chunk) units of all
// pairs, pair-major, are cut into equal contiguous ranges, one per
// attention warp of the grid (stream-K, as for the projections), so every
// warp reads the same number of cache bytes.  A warp streams its chunks
// through two shared buffers of its own (bulk copies; the next chunk in
// flight while one is computed; the first chunk of each pair brings the
// pair's query along).  Within a chunk each group of 8 lanes takes every 4th
// key: all its scores first (independent dot products), then one rescale of
// the running (max, sum, output) by the chunk maximum, then the weighted
// values.  Where a warp's range leaves a pair, the four groups merge with
// shuffles; a pair inside one range is written directly, otherwise each
// range leaves its (max, sum, output) in the workspace and the last range to
// arrive merges them in range order.
// Chunk kc of query pair pr = b * H + h, whose keys and values are cache row
// kvr = b * Hkv + h / (H / Hkv); PG: the cache is paged (the kernel is
// instantiated apart for paged and contiguous caches).
template <int BN, int HD, bool PG>
__device__ __forceinline__ void attn_issue_kv(const StepArgs& a, int l, int b, int kvr, int kc, int len, uint32_t dst,
                                              uint32_t bar, uint32_t extra_bytes, bool arrive) {
    const int k0 = kc * ACH;
    const int nkeys = min(len - k0, ACH);
    const bf16* kc_ = a.kv + (size_t)(2 * l) * a.kv_layer;
    const bf16* vc = kc_ + a.kv_layer;
    // a chunk never crosses a page of a paged cache (ACH divides KV_PAGE)
    const size_t off = kv_row_offset(PG ? a.pages : nullptr, a.pps, b, a.Hkv, kvr - b * a.Hkv, a.smax, k0, HD);
    const uint32_t bytes = (uint32_t)(nkeys * HD * 2);
    // cache rows are read once per step (per query head of a group): first out of L2
    const uint64_t pol = l2_evict_first();
    if (arrive)
        mbar_expect_tx(bar, 2 * bytes + extra_bytes);
    else   // the barrier's one arrival comes later, with the query (or without it)
        asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(2 * bytes)
                     : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
            "r"(dst),
        "l"(kc_ + off), "r"(bytes), "r"(bar), "l"(pol)
        : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
            "r"(dst + ACH * HD * 2),
        "l"(vc + off), "r"(bytes), "r"(bar), "l"(pol)
        : "memory");
}
template <int BN, int HD>
__device__ __forceinline__ void attn_issue_q(const StepArgs& a, int pr, uint32_t dst, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     dst + SCfg<BN, HD>::ATT_Q),
                 "l"(a.q + (size_t)pr * HD), "r"((uint32_t)(HD * 2)), "r"(bar)
                 : "memory");
}

// Attention of layer l for attention warp aw of this CTA (0..NAW-1).
template <int BN, int HD, bool PG>
__device__ bool phase_attn(const StepArgs& a, int l, int aw, int lane, const Smem<BN, HD>& sm, uint32_t* uses,
                           volatile int* abort_flag) {
    using C = SCfg<BN, HD>;
    constexpr int DPL = HD / 8;      // dims per lane: 16-byte vectors u, dims (u*8 + r)*8 ..
    constexpr int NV = DPL / 8;
    constexpr int KPG = ACH / 4;     // keys of a chunk per lane group
    constexpr int DPW = HD / 32;     // dims per lane in the final merge
    const int g = lane >> 3, r = lane & 7;
    // Sequence j (lane j) holds len_j = pos_j + 1 keys in n_j chunks; the
    // chunks of all pairs, pair-major (pair = j * H + h), form one range of
    // H * sum_j n_j units whose sequence j starts at H * (n_0 + ... + n_{j-1}).
    const int Bq = a.B;
    const int my_len = lane < Bq ? a.d_pos[lane] + 1 : 0;
    const int my_nch = (my_len + ACH - 1) / ACH;
    int incl = my_nch;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    const int excl = incl - my_nch;
    const long long Ctot = (long long)a.H * __shfl_sync(0xffffffffu, incl, Bq - 1);
    const int Wp = (int)min((long long)gridDim.x * NAW, Ctot);
    const int gw = blockIdx.x * NAW + aw;
    if (gw >= Wp) {
        // no attention work here: still wait for this layer's QKV count, so
        // that attention warps 6 and 7 arrive at the named barrier they share
        // with the epilogue warps once per layer, never a layer ahead
        int w = 1;
        if (lane == 0) {
            unsigned tgt = 0;
            const unsigned* dp = dep_of(a, PH_ATTN, l, tgt);
            w = wait_at_least(dp, tgt, abort_flag, a.err);
        }
        return __shfl_sync(0xffffffffu, w, 0) != 0;
    }
    const long long cs = Ctot * gw / Wp, ce = Ctot * (gw + 1) / Wp;
    auto owner = [&](long long i) { return (int)(((i + 1) * Wp - 1) / Ctot); };
    // unit index -> (sequence b, head h, chunk kc) with b's length and chunk
    // count; the key/value row kvr = b * Hkv + h / G follows h without a division
    const int G = a.H / a.Hkv;
    struct Pos {
        int b, h, kc, len, nch, kvr, hg;
    };
    auto locate = [&](long long c) {
        Pos q;
        q.b = __popc(__ballot_sync(0xffffffffu, lane < Bq && (long long)a.H * incl <= c));
        q.len = __shfl_sync(0xffffffffu, my_len, q.b);
        q.nch = __shfl_sync(0xffffffffu, my_nch, q.b);
        const long long rem = c - (long long)a.H * __shfl_sync(0xffffffffu, excl, q.b);
        q.h = (int)(rem / q.nch);
        q.kc = (int)(rem - (long long)q.h * q.nch);
        q.kvr = q.b * a.Hkv + q.h / G;
        q.hg = q.h % G;
        return q;
    };
    auto advance = [&](Pos& q) {
        if (++q.kc < q.nch) return;
        q.kc = 0;
        if (++q.hg == G) {        // the next key/value head (also across sequences: rows are b * Hkv + ...)
            q.hg = 0;
            ++q.kvr;
        }
        if (++q.h < a.H) return;
        q.h = 0;
        ++q.b;
        const int bb = min(q.b, 31);
        q.len = __shfl_sync(0xffffffffu, my_len, bb);
        q.nch = __shfl_sync(0xffffffffu, my_nch, bb);
    };
    const uint32_t wbuf = smem_u32(sm.att) + aw * 2 * C::ATT_BUF;
    const uint32_t wbar = sm.abar + aw * 16;
    // issue cursor
    long long ic = cs;
    Pos iq = locate(cs);
    auto issue = [&](int buf) {
        if (lane == 0) {
            const bool with_q = ic == cs || iq.kc == 0;
            const uint32_t dst = wbuf + buf * C::ATT_BUF, bar = wbar + 8 * buf;
            attn_issue_kv<BN, HD, PG>(a, l, iq.b, iq.kvr, iq.kc, iq.len, dst, bar, with_q ? HD * 2 : 0, true);
            if (with_q) attn_issue_q<BN, HD>(a, iq.b * a.H + iq.h, dst, bar);
        }
        ++ic;
        advance(iq);
    };
    // The first two chunks' keys and values go out before this layer's QKV
    // projection is complete, unless a chunk holds the position this step
    // appends (its pair's last chunk): those rows were written by earlier
    // steps.  Their query (and their one barrier arrival) follows once the
    // QKV count is complete.  Shared memory first: its earlier generic
    // writes (the epilogues' transpose buffer) before the async copies.
    if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    bool early[2] = {false, false};
    {
        Pos eq = iq;
        for (int k = 0; k < 2 && cs + k < ce; ++k) {
            early[k] = eq.kc < eq.nch - 1;
            if (early[k] && lane == 0)
                attn_issue_kv<BN, HD, PG>(a, l, eq.b, eq.kvr, eq.kc, eq.len, wbuf + k * C::ATT_BUF, wbar + 8 * k, 0,
                                      false);
            advance(eq);
        }
    }
    // this layer's QKV projection complete (queries, and the newest keys and values)
    {
        int w = 1;
        if (lane == 0) {
            unsigned tgt = 0;
            const unsigned* dp = dep_of(a, PH_ATTN, l, tgt);
            w = wait_at_least(dp, tgt, abort_flag, a.err);
        }
        if (!__shfl_sync(0xffffffffu, w, 0)) {
            // leave no early copy in flight: arrive, then wait (bounded) for the bytes
            if (lane == 0)
                for (int k = 0; k < 2; ++k)
                    if (early[k]) {
                        mbar_arrive(wbar + 8 * k);
                        const uint64_t t0 = global_timer();
                        while (!mbar_try_wait(wbar + 8 * k, uses[k] & 1u) &&
                               global_timer() - t0 < WAIT_LIMIT_NS / 4) {
                        }
                        uses[k]++;
                    }
            __syncwarp();
            return false;
        }
    }
    // the queries and the newest cache rows of this step were stored by other
    // CTAs (generic proxy) before their completion counts; the bulk copies
    // read them through the async proxy
    if (lane == 0) asm volatile("fence.proxy.async.global;" ::: "memory");
    __syncwarp();
    for (int k = 0; k < 2 && ic < ce; ++k) {
        if (early[k]) {
            if (lane == 0) {
                const uint32_t dst = wbuf + k * C::ATT_BUF, bar = wbar + 8 * k;
                if (ic == cs || iq.kc == 0) {
                    mbar_expect_tx(bar, HD * 2);
                    attn_issue_q<BN, HD>(a, iq.b * a.H + iq.h, dst, bar);
                } else {
                    mbar_arrive(bar);
                }
            }
            ++ic;
            advance(iq);
        } else {
            issue(k);
        }
    }
    const float scale = rsqrtf((float)HD);
    float m = -INFINITY, lsum = 0.f, acc[DPL], qv[DPL];
    Pos cq = locate(cs);
    for (long long c = cs; c < ce; ++c) {
        const int k = (int)(c - cs), buf = k & 1;
        const uint32_t bar = wbar + 8 * buf;
        bool ok = false;
        {
            const uint64_t t0 = global_timer();
            while (true) {
                if (mbar_try_wait(bar, uses[buf] & 1u)) {
                    ok = true;
                    break;
                }
                if (*abort_flag || global_timer() - t0 > WAIT_LIMIT_NS) break;
            }
        }
        uses[buf]++;
        if (__any_sync(0xffffffffu, !ok)) {
            if (lane == 0) {
                *abort_flag = 1;
                atomicOr(a.err, LLAMA_DEVERR_TIMEOUT);
            }
            return false;
        }
        const uint8_t* bp = sm.att + (size_t)(aw * 2 + buf) * C::ATT_BUF;
        const bf16* sk = reinterpret_cast<const bf16*>(bp);
        const bf16* sv = sk + ACH * HD;
        const int kc = cq.kc, nch = cq.nch, len = cq.len;
        if (c == cs || kc == 0) {    // a new pair: its query (in this buffer) and a fresh state
            const bf16* qp = reinterpret_cast<const bf16*>(bp + C::ATT_Q);
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                const uint4 w = *reinterpret_cast<const uint4*>(qp + (u * 8 + r) * 8);
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float2 f = unpack_bf16x2(ws[t]);
                    qv[u * 8 + 2 * t] = f.x * scale;
                    qv[u * 8 + 2 * t + 1] = f.y * scale;
                }
            }
            m = -INFINITY;
            lsum = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
        }
        const int nkeys = min(len - kc * ACH, ACH);
        // scores of this group's keys 4i + g (row 0 stands in for a missing key)
        float s[KPG];
#pragma unroll
        for (int i = 0; i < KPG; ++i) {
            const int key = 4 * i + g;
            const int kr = key < nkeys ? key : 0;
            float d0 = 0.f, d1 = 0.f;
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                const uint4 wk = *reinterpret_cast<const uint4*>(sk + (size_t)kr * HD + (u * 8 + r) * 8);
                const uint32_t k4[4] = {wk.x, wk.y, wk.z, wk.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float2 fk = unpack_bf16x2(k4[t]);
                    d0 = fmaf(qv[u * 8 + 2 * t], fk.x, d0);
                    d1 = fmaf(qv[u * 8 + 2 * t + 1], fk.y, d1);
                }
            }
            s[i] = d0 + d1;
        }
#pragma unroll
        for (int off = 1; off <= 4; off <<= 1)
#pragma unroll
            for (int i = 0; i < KPG; ++i) s[i] += __shfl_xor_sync(0xffffffffu, s[i], off);
        float cmax = -INFINITY;
#pragma unroll
        for (int i = 0; i < KPG; ++i)
            if (4 * i + g < nkeys) cmax = fmaxf(cmax, s[i]);
        const float m_new = fmaxf(m, cmax);
        if (m_new != -INFINITY) {   // this group holds at least one key so far
            const float corr = __expf(m - m_new);
            float pk[KPG], psum = 0.f;
#pragma unroll
            for (int i = 0; i < KPG; ++i) {
                pk[i] = (4 * i + g < nkeys) ? __expf(s[i] - m_new) : 0.f;
                psum += pk[i];
            }
            lsum = lsum * corr + psum;
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[e] *= corr;
#pragma unroll
            for (int i = 0; i < KPG; ++i) {
                const int key = 4 * i + g;
                const int kr = key < nkeys ? key : 0;
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                    const uint4 wv = *reinterpret_cast<const uint4*>(sv + (size_t)kr * HD + (u * 8 + r) * 8);
                    const uint32_t v4[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const float2 fv = unpack_bf16x2(v4[t]);
                        acc[u * 8 + 2 * t] = fmaf(pk[i], fv.x, acc[u * 8 + 2 * t]);
                        acc[u * 8 + 2 * t + 1] = fmaf(pk[i], fv.y, acc[u * 8 + 2 * t + 1]);
                    }
                }
            }
            m = m_new;
        }
        __syncwarp();
        // the buffer is free: put the chunk two places ahead in flight
        if (ic < ce) issue(buf);
        const int pb = cq.b, ph = cq.h, pr = pb * a.H + ph;
        const bool pair_done = (c + 1 == ce) || (kc + 1 == nch);
        advance(cq);
        if (!pair_done) continue;
        // merge the four lane groups (each covers every 4th key)
#pragma unroll
        for (int off = 8; off <= 16; off <<= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
            const float l2 = __shfl_xor_sync(0xffffffffu, lsum, off);
            const float M = fmaxf(m, m2);
            const float c1 = (m == -INFINITY) ? 0.f : __expf(m - M);
            const float c2 = (m2 == -INFINITY) ? 0.f : __expf(m2 - M);
            lsum = lsum * c1 + l2 * c2;
#pragma unroll
            for (int e = 0; e < DPL; ++e) {
                const float o2 = __shfl_xor_sync(0xffffffffu, acc[e], off);
                acc[e] = acc[e] * c1 + o2 * c2;
            }
            m = M;
        }
        const long long pc0 = (long long)a.H * __shfl_sync(0xffffffffu, excl, pb) + (long long)ph * nch;
        const int first = owner(pc0), nparts = owner(pc0 + nch - 1) - first + 1;
        bf16* dst = a.attn + (size_t)pb * a.d + (size_t)ph * HD;
        if (nparts == 1) {    // the whole pair in this range
            const float inv = 1.f / lsum;
            if (g == 0) {
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                    uint4 o;
                    o.x = pack_bf16x2(acc[u * 8 + 0] * inv, acc[u * 8 + 1] * inv);
                    o.y = pack_bf16x2(acc[u * 8 + 2] * inv, acc[u * 8 + 3] * inv);
                    o.z = pack_bf16x2(acc[u * 8 + 4] * inv, acc[u * 8 + 5] * inv);
                    o.w = pack_bf16x2(acc[u * 8 + 6] * inv, acc[u * 8 + 7] * inv);
                    *reinterpret_cast<uint4*>(dst + (u * 8 + r) * 8) = o;
                }
            }
            __syncwarp();
            if (lane == 0) count_done(done_ctr(a, l, DK_ATTN));
            continue;
        }
        float* wp = a.attn_work + ((size_t)gw + pr) * (HD + 2);
        if (g == 0) {
#pragma unroll
            for (int u = 0; u < NV; ++u)
#pragma unroll
                for (int t = 0; t < 8; ++t) wp[2 + (u * 8 + r) * 8 + t] = acc[u * 8 + t];
            if (r == 0) {
                wp[0] = m;
                wp[1] = lsum;
            }
        }
        __syncwarp();
        int last = 0;
        if (lane == 0) {
            const int prev = arrive_acq_rel(a.attn_cnt + pr);
            last = (prev == nparts - 1);
            if (last) a.attn_cnt[pr] = 0;   // published by this warp's later release
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) continue;
        const float* wb = a.attn_work + ((size_t)first + pr) * (HD + 2);
        // lane j owns range j (and j + 32, ...): maxima and weighted sums by shuffles
        float Mall = -INFINITY;
        for (int j = lane; j < nparts; j += 32) Mall = fmaxf(Mall, __ldcg(wb + (size_t)j * (HD + 2)));
        Mall = warp_max(Mall);
        float L = 0.f, o[DPW];
#pragma unroll
        for (int e = 0; e < DPW; ++e) o[e] = 0.f;
        for (int j0 = 0; j0 < nparts; j0 += 32) {
            const int j = j0 + lane;
            float w = 0.f;
            if (j < nparts) {
                const float mj = __ldcg(wb + (size_t)j * (HD + 2));
                w = (mj == -INFINITY) ? 0.f : __expf(mj - Mall);
                L += __ldcg(wb + (size_t)j * (HD + 2) + 1) * w;
            }
            const int jn = min(32, nparts - j0);
#pragma unroll 4
            for (int t = 0; t < jn; ++t) {
                const float wt = __shfl_sync(0xffffffffu, w, t);
                const float* pc = wb + (size_t)(j0 + t) * (HD + 2) + 2 + lane * DPW;
#pragma unroll
                for (int e = 0; e < DPW; ++e) o[e] = fmaf(__ldcg(pc + e), wt, o[e]);
            }
        }
        L = warp_sum(L);
        const float inv = 1.f / L;
#pragma unroll
        for (int e = 0; e < DPW; ++e) dst[lane * DPW + e] = __float2bfloat16_rn(o[e] * inv);
        __syncwarp();
        if (lane == 0) count_done(done_ctr(a, l, DK_ATTN));
    }
    return true;
}

// ---------------------------------------------------------------- greedy choice
__device__ bool amx_better(float v, int i, float bv, int bi) { return v > bv || (v == bv && i < bi); }

template <int BN, int HD>
__device__ void phase_argmax(const StepArgs& a, int tid, const Smem<BN, HD>& sm, unsigned E, volatile int* abort_flag) {
    const int nc = (a.V + AMX - 1) / AMX;
    const int nitems = a.B * nc;
    int* sidx = reinterpret_cast<int*>(sm.red + 8);
    for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
        const int b = item / nc, c = item - b * nc;
        const float* p = a.logits + (size_t)b * a.V;
        float best = -INFINITY;
        int bi = 0x7fffffff;
        for (int i = c * AMX + tid; i < min(a.V, (c + 1) * AMX); i += 128) {
            const float v = __ldcg(p + i);
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
        if ((tid & 31) == 0) {
            sm.red[tid >> 5] = best;
            sidx[tid >> 5] = bi;
        }
        esync();
        if (tid == 0) {
            for (int k = 1; k < 4; ++k)
                if (amx_better(sm.red[k], sidx[k], best, bi)) {
                    best = sm.red[k];
                    bi = sidx[k];
                }
            a.amax_part[(size_t)b * nc + c] = make_int2(__float_as_int(best), bi);
            __threadfence();
            const int prev = atomicAdd(a.amax_cnt + b, 1);
            if (prev == nc - 1) {
                a.amax_cnt[b] = 0;
                __threadfence();
                float fb = -INFINITY;
                int fi = 0x7fffffff;
                for (int k = 0; k < nc; ++k) {
                    const int2 e = __ldcg(a.amax_part + (size_t)b * nc + k);
                    if (amx_better(__int_as_float(e.x), e.y, fb, fi)) {
                        fb = __int_as_float(e.x);
                        fi = e.y;
                    }
                }
                a.tok[b] = (fi == 0x7fffffff) ? 0 : fi;
                // the last row to finish advances the position
                __threadfence();
                const int rows = atomicAdd(a.amax_cnt + a.B, 1);
                if (rows == a.B - 1) {
                    a.amax_cnt[a.B] = 0;
                    // close the step once every CTA has started it (and so
                    // has read its epoch)
                    wait_at_least(a.bar + SY_CHECKIN, gridDim.x, abort_flag, a.err);
                    a.bar[SY_CHECKIN] = 0;
                    a.bar[SY_EPOCH] = E;
                    for (int j = 0; j < a.B; ++j) a.d_pos[j] += 1;
                }
            }
        }
        esync();
    }
}


// ---------------------------------------------------------------- the kernel
template <int BN, int HD, bool PG>
__global__ void __launch_bounds__(NT, 1) decode_step_kernel(StepArgs a) {
    using C = SCfg<BN, HD>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base_s = (raw + 1023u) & ~1023u;
    uint8_t* gb = smem_raw + (base_s - raw);
    Smem<BN, HD> sm;
    sm.sA = base_s + C::OFF_A;
    sm.sB = base_s + C::OFF_B;
    sm.att = gb + C::OFF_ATT;
    sm.xbuf = reinterpret_cast<float*>(gb + C::OFF_X);
    sm.sinv = reinterpret_cast<float*>(gb + C::OFF_SML);
    sm.red = sm.sinv + 32;
    const uint32_t bars = base_s + C::OFF_BAR;
    sm.full = bars;
    sm.empty = bars + 8 * C::STAGES;
    sm.tfull = bars + 16 * C::STAGES;
    sm.tempty = sm.tfull + 16;
    sm.abar = sm.tempty + 16;                                       // [NAW warps][2]
    uint32_t* misc = reinterpret_cast<uint32_t*>(gb + C::OFF_MISC);
    uint32_t* tmem_slot = misc;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    sm.flag = reinterpret_cast<volatile int*>(misc + 2);
    volatile unsigned* epoch = reinterpret_cast<volatile unsigned*>(misc + 3);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = phase_count(a);
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(sm.full + 8 * s, 1);
            mbar_init(sm.empty + 8 * s, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(sm.tfull + 8 * i, 1);
            mbar_init(sm.tempty + 8 * i, 128);
        }
        for (int i = 0; i < 2 * NAW; ++i) mbar_init(sm.abar + 8 * i, 1);
        *abort_flag = 0;
        // this step's epoch; the step is closed (and the word advanced) only
        // after every CTA has checked in here
        *epoch = ld_acquire_u32(a.bar + SY_EPOCH) + 1u;
        atomicAdd(a.bar + SY_CHECKIN, 1u);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const unsigned E = *epoch;

    if (warp == 4) {
        // -------------------------------------------------------- TMA producer
        // Two cursors over the same stage sequence: weight tiles are requested
        // as soon as a ring slot frees; the activation tile of a stage only
        // once the completion count its phase reads after is complete.
        if (lane == 0) {
            Cursor wc, xc;
            cursor_seek(a, P, wc, 0);
            xc = wc;
            int wn = 0, xn = 0, ready = -1;
            const uint64_t wpol = l2_evict_first();   // a weight tile is read once per step
            // the embedding (and the reset of the completion counts) first
            bool ok0 = wait_at_least(a.bar + SY_EMBED, E, abort_flag, a.err);
            uint64_t t_last = global_timer();
            while (xc.valid && ok0) {
                bool prog = false;
                if (wc.valid && wn - xn < C::STAGES) {
                    const int slot = wn % C::STAGES;
                    if (mbar_test(sm.empty + 8 * slot, ((wn / C::STAGES) & 1) ^ 1)) {
                        mbar_expect_tx(sm.full + 8 * slot, C::STAGE_BYTES);
                        tma_load_2d_hint(sm.sA + slot * C::A_BYTES, a.maps + wc.map_a, sm.full + 8 * slot, wc.kb * BK,
                                         wc.mb * BM, wpol);
                        ++wn;
                        cursor_next(a, P, wc);
                        prog = true;
                    }
                }
                if (xn < wn) {
                    if (ready < xc.p && (!xc.dep || (int)(ld_acquire_u32(xc.dep) - xc.tgt) >= 0)) {
                        asm volatile("fence.proxy.async.global;" ::: "memory");
                        ready = xc.p;
                    }
                    if (ready >= xc.p) {
                        const int slot = xn % C::STAGES;
                        tma_load_2d(sm.sB + slot * C::B_BYTES, a.maps + xc.map_b, sm.full + 8 * slot, xc.kb * BK, 0);
                        ++xn;
                        cursor_next(a, P, xc);
                        prog = true;
                    }
                }
                if (prog) {
                    t_last = global_timer();
                    continue;
                }
                if (*abort_flag) break;
                if (global_timer() - t_last > WAIT_LIMIT_NS) {
                    *abort_flag = 1;
                    atomicOr(a.err, LLAMA_DEVERR_TIMEOUT);
                    break;
                }
                __nanosleep(32);   // leave issue slots to the epilogue warp on this sub-partition
            }
            // Leave no copy in flight: complete every stage whose weight tile
            // was requested (its activation tile too, stale or not, so that its
            // barrier can complete), then wait -- bounded -- for the last ring
            // of stages to land.
            while (xn < wn) {
                const int slot = xn % C::STAGES;
                tma_load_2d(sm.sB + slot * C::B_BYTES, a.maps + xc.map_b, sm.full + 8 * slot, xc.kb * BK, 0);
                ++xn;
                cursor_next(a, P, xc);
            }
            for (int u = max(0, wn - C::STAGES); u < wn; ++u) {
                const uint64_t t0 = global_timer();
                while (!mbar_test(sm.full + 8 * (u % C::STAGES), (u / C::STAGES) & 1) &&
                       global_timer() - t0 < WAIT_LIMIT_NS / 4) {
                }
            }
        }
    } else if (warp == 5) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_bf16(BN);
            int stage = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t acc_ph = 0;
            bool ok = true;
            for (int p = 0; p < P && ok; ++p) {
                int l;
                const int type = phase_type(a, p, l);
                Work w;
                if (!work_of(a, type, l, w)) continue;
                for (int i = w.s; i < w.e && ok;) {
                    const int se = min(w.e, (i / w.kbt + 1) * w.kbt);   // end of this block's run
                    if (!mbar_wait(sm.tempty + 8 * acc, acc_ph ^ 1u, abort_flag, a.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
                    for (int it = i; it < se; ++it) {
                        if (!mbar_wait(sm.full + 8 * stage, ph, abort_flag, a.err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t da = sw128_desc(sm.sA + stage * C::A_BYTES);
                        const uint64_t db = sw128_desc(sm.sB + stage * C::B_BYTES);
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k)
                            umma_bf16(d_tmem, da + 2 * k, db + 2 * k, IDESC, (it > i || k > 0) ? 1u : 0u);
                        umma_commit(sm.empty + 8 * stage);
                        if (++stage == C::STAGES) {
                            stage = 0;
                            ph ^= 1u;
                        }
                    }
                    if (!ok) break;
                    umma_commit(sm.tfull + 8 * acc);
                    if (++acc == 2) {
                        acc = 0;
                        acc_ph ^= 1u;
                    }
                    i = se;
                }
            }
        }
    } else if (warp < 4) {
        // -------------------------------------------------------- epilogue warps 0..3
        const int tid = threadIdx.x;
        const int quarter = warp;
        const int et = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        int acc = 0;
        uint32_t acc_ph = 0;
        uint32_t uses[2] = {0u, 0u};
        unsigned long long* tl = a.timeline ? a.timeline + (size_t)blockIdx.x * P * 2 : nullptr;
        for (int p = 0; p < P; ++p) {
            int l;
            const int type = phase_type(a, p, l);
            {
                // wait for this phase's input (its completion count; before
                // the first projection also the embedding, which zeroes the
                // counts)
                bool ok = true;
                if (tid == 0) {
                    unsigned tgt = 0;
                    // attention: each attention warp waits itself, after its first copies
                    const unsigned* dp = (type == PH_EMBED || type == PH_ATTN) ? nullptr : dep_of(a, type, l, tgt);
                    if (dp) ok = wait_at_least(dp, tgt, abort_flag, a.err);
                    // the embedding (and the zeroed counts) before anything else
                    if (ok && p == 1) ok = wait_at_least(a.bar + SY_EMBED, E, abort_flag, a.err);
                }
                if (esync_any(!ok)) break;
            }
            if (tl && tid == 0) tl[2 * p] = global_timer();
            bool fail = false;
            if (type == PH_EMBED) {
                // CTA b < B: the embedding of row b's token, bf16(g * x) of
                // the first attention norm and the row's 128-feature block
                // sums of squares (one warp per block: 32 lanes x 4
                // features).  The last row to finish zeroes the completion
                // counts of this step and publishes its epoch.
                if ((int)blockIdx.x < a.B) {
                    const int b = blockIdx.x;
                    int t = a.tok[b];
                    if (t < 0 || t >= a.V) {
                        if (tid == 0) atomicOr(a.err, 2);
                        t = 0;
                    }
                    const bf16* e = a.embed + (size_t)t * a.d;
                    float* x = a.trunk + (size_t)b * a.d;
                    const float* g0 = a.gains[0];
                    for (int i = 4 * tid; i < a.d; i += 512) {
                        const uint2 w = *reinterpret_cast<const uint2*>(e + i);
                        const float2 v01 = unpack_bf16x2(w.x), v23 = unpack_bf16x2(w.y);
                        const float4 gg = *reinterpret_cast<const float4*>(g0 + i);
                        *reinterpret_cast<float4*>(x + i) = make_float4(v01.x, v01.y, v23.x, v23.y);
                        *reinterpret_cast<uint2*>(a.xg + (size_t)b * a.d + i) =
                            make_uint2(pack_bf16x2(v01.x * gg.x, v01.y * gg.y), pack_bf16x2(v23.x * gg.z, v23.y * gg.w));
                        const float s = warp_sum((v01.x * v01.x + v01.y * v01.y) + (v23.x * v23.x + v23.y * v23.y));
                        if (lane == 0) a.ssq[(i >> 7) * 32 + b] = s;
                    }
                    esync();
                    int last = 0;
                    if (tid == 0) {
                        __threadfence();
                        const unsigned prev = atomicAdd(a.bar + SY_ROWS, 1u);
                        last = (prev == (unsigned)a.B - 1u);
                        if (last) a.bar[SY_ROWS] = 0u;
                    }
                    if (esync_any(last)) {
                        for (int i = tid; i < 8 * (a.L + 1); i += 128) a.bar[SY_DONE + 32 * i] = 0u;
                        esync();
                        if (tid == 0) {
                            __threadfence();
                            asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(a.bar + SY_EMBED), "r"(E)
                                         : "memory");
                        }
                    }
                }
            } else if (type == PH_ATTN) {
                fail = !phase_attn<BN, HD, PG>(a, l, warp, lane, sm, uses, abort_flag);
                asm volatile("bar.sync 2, 192;" ::: "memory");   // with attention warps 6, 7
            } else if (type == PH_ARGMAX) {
                phase_argmax<BN, HD>(a, tid, sm, E, abort_flag);
            } else {
                Work w;
                work_of(a, type, l, w);
                if (type == PH_QKV || type == PH_HEAD) load_inv(a, a.ssq, sm.sinv, tid);
                else if (type == PH_GU) load_inv(a, a.ssq + SSQ_BLOCKS * 32, sm.sinv, tid);
                EpiArgs ep;
                memset(&ep, 0, sizeof(ep));
                ep.M = a.B;
                ep.N = w.g.rowsA;
                ep.out = (type == PH_HEAD) ? a.logits : a.trunk;
                ep.ld_out = (type == PH_HEAD) ? a.V : a.d;
                ep.partial = a.partial;
                ep.counters = a.counters;
                ep.act = a.act;
                ep.hidden = a.h;
                ep.q = a.q;
                ep.kc = a.kv + (size_t)(2 * l) * a.kv_layer;
                ep.vc = a.kv + (size_t)(2 * l + 1) * a.kv_layer;
                ep.rope = a.rope;
                ep.d_pos = a.d_pos;
                ep.S = 1;
                ep.H = a.H;
                ep.hd = a.hd;
                ep.d = a.d;
                ep.smax = a.smax;
                ep.Hkv = a.Hkv;
                ep.pages = PG ? a.pages : nullptr;
                ep.pps = a.pps;
                ep.bias = (type == PH_QKV && a.biases) ? a.biases[4 * l] : nullptr;   // folded QKV biases
                for (int i = w.s; i < w.e;) {
                    const int mb = i / w.kbt;
                    const bool ok = mbar_wait(sm.tfull + 8 * acc, acc_ph, abort_flag, a.err);
                    if (esync_any(!ok)) {
                        fail = true;
                        break;
                    }
                    tc_fence_after();
                    float v[32];
                    const uint32_t tacc = tmem + lane_addr + (uint32_t)(acc * BN);
                    if constexpr (BN == 16) tmem_ld16(tacc, v);
                    else tmem_ld32(tacc, v);
                    tc_fence_before();
                    mbar_arrive(sm.tempty + 8 * acc);
                    if (++acc == 2) {
                        acc = 0;
                        acc_ph ^= 1u;
                    }
                    switch (w.g.mode) {
                        case EPI_QKV: tile_epilogue<BN, HD, EPI_QKV>(a, ep, w, l, type, mb, et, tid, v, sm); break;
                        case EPI_RESID: tile_epilogue<BN, HD, EPI_RESID>(a, ep, w, l, type, mb, et, tid, v, sm); break;
                        case EPI_SWIGLU: tile_epilogue<BN, HD, EPI_SWIGLU>(a, ep, w, l, type, mb, et, tid, v, sm); break;
                        default: tile_epilogue<BN, HD, EPI_F32>(a, ep, w, l, type, mb, et, tid, v, sm); break;
                    }
                    i = min(w.e, (mb + 1) * w.kbt);
                }
            }
            if (esync_any(fail)) break;
            if (tl && tid == 0) tl[2 * p + 1] = global_timer();
        }
    } else {
        // -------------------------------------------------------- attention warps 6, 7
        // They join the epilogue warps in each attention phase: wait for the
        // QKV completion count that opens it, take their share, and arrive at
        // the named barrier the epilogue warps pass before they leave the
        // phase (once per layer, also after a failure, so that nobody waits
        // for them).
        uint32_t uses[2] = {0u, 0u};
        int w = 1;
        if (lane == 0) w = wait_at_least(a.bar + SY_EMBED, E, abort_flag, a.err);
        bool ok = __shfl_sync(0xffffffffu, w, 0) != 0;
        for (int l = 0; l < a.L; ++l) {
            if (ok) ok = phase_attn<BN, HD, PG>(a, l, warp - 2, lane, sm, uses, abort_flag);
            __syncwarp();
            asm volatile("bar.arrive 2, 192;" ::: "memory");
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                     : "memory");
    }
}

template <int BN, int HD, bool PG>
int launch_step_t(const StepArgs& a, cudaStream_t st) {
    using C = SCfg<BN, HD>;
    static PerDeviceOnce once;
    int rc = once_per_device(once, []() -> int {
        LLAMA_CUDA_TRY(cudaFuncSetAttribute(decode_step_kernel<BN, HD, PG>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
        return (int)LLAMA_OK;
    });
    if (rc) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(decode_step_ctas());
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr_c[1];
    attr_c[0].id = cudaLaunchAttributeCooperative;
    attr_c[0].val.cooperative = 1;
    cfg.attrs = attr_c;
    cfg.numAttrs = 1;
    LLAMA_CUDA_TRY(cudaLaunchKernelEx(&cfg, decode_step_kernel<BN, HD, PG>, a));
    llama_count_launches(1);
    return LLAMA_OK;
}

}  // namespace

int decode_step_ctas() { return std::min(tc_num_sms(), STEP_MAX_CTAS); }

// Partial-sum and counter regions of the five projection kinds (qkv, o,
// gate/up, down, head) for `ctas` CTAs and batch B; returns the floats of
// all partial regions.
long long decode_step_layout(int ctas, int qkv_rows, int d, int h, int V, int B, long long part_off[5],
                             int cnt_off[5]) {
    const int rows[5] = {qkv_rows, d, 2 * h, d, V};
    const long long Mp = (B + 3) & ~3;
    long long off = 0;
    int coff = 0;
    for (int t = 0; t < 5; ++t) {
        const int mblk = rows[t] / BM;
        part_off[t] = off;
        off += (long long)rows[t] * step_slots(mblk, ctas) * Mp;
        cnt_off[t] = coff;
        coff += (t == 2) ? mblk / 2 : mblk;
    }
    return off;
}

template <int BN, int HD>
int step_prepare_t() {
    LLAMA_CUDA_TRY(cudaFuncSetAttribute(decode_step_kernel<BN, HD, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        SCfg<BN, HD>::SMEM));
    LLAMA_CUDA_TRY(cudaFuncSetAttribute(decode_step_kernel<BN, HD, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        SCfg<BN, HD>::SMEM));
    return LLAMA_OK;
}

int decode_step_prepare() {
    int n = 0;
    if (int rc = step_prepare_t<16, 128>()) return rc;
    if (int rc = step_prepare_t<32, 128>()) return rc;
    if (int rc = step_prepare_t<16, 64>()) return rc;
    if (int rc = step_prepare_t<32, 64>()) return rc;
    // one CTA per SM must fit for the cooperative launch
    LLAMA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_step_kernel<16, 128, false>, NT,
                                                                 SCfg<16, 128>::SMEM));
    return n >= 1 ? LLAMA_OK : LLAMA_ERR_CUDA;
}

int launch_decode_step(const StepArgs& a, cudaStream_t st) {
    if (a.B <= 0 || a.B > 32) return LLAMA_ERR_INVALID_ARG;
    const bool pg = a.pages != nullptr;
    if (a.hd == 128)
        return a.B <= 16 ? (pg ? launch_step_t<16, 128, true>(a, st) : launch_step_t<16, 128, false>(a, st))
                         : (pg ? launch_step_t<32, 128, true>(a, st) : launch_step_t<32, 128, false>(a, st));
    if (a.hd == 64)
        return a.B <= 16 ? (pg ? launch_step_t<16, 64, true>(a, st) : launch_step_t<16, 64, false>(a, st))
                         : (pg ? launch_step_t<32, 64, true>(a, st) : launch_step_t<32, 64, false>(a, st));
    return LLAMA_ERR_INVALID_ARG;
}

// Tensor-map table for the decode step: 4 per layer (W_qkv, W_o, W_gu, W_d),
// the head, then the activation buffers xg, attn, act, xg2 with `B` rows.
int decode_step_maps(CUtensorMap* host_maps, const void* const* w, int L, const void* head, const void* xg,
                     const void* attn, const void* act, const void* xg2, int B, int qkv_rows, int d, int h, int V) {
    int rc;
    const int bn = B <= 16 ? 16 : 32;
    for (int l = 0; l < L; ++l) {
        if ((rc = tc_make_map_2d(&host_maps[4 * l + 0], w[4 * l + 0], qkv_rows, d, BM))) return rc;
        if ((rc = tc_make_map_2d(&host_maps[4 * l + 1], w[4 * l + 1], d, d, BM))) return rc;
        if ((rc = tc_make_map_2d(&host_maps[4 * l + 2], w[4 * l + 2], 2 * h, d, BM))) return rc;
        if ((rc = tc_make_map_2d(&host_maps[4 * l + 3], w[4 * l + 3], d, h, BM))) return rc;
    }
    if ((rc = tc_make_map_2d(&host_maps[4 * L + 0], head, V, d, BM))) return rc;
    if ((rc = tc_make_map_2d(&host_maps[4 * L + 1], xg, B, d, bn))) return rc;
    if ((rc = tc_make_map_2d(&host_maps[4 * L + 2], attn, B, d, bn))) return rc;
    if ((rc = tc_make_map_2d(&host_maps[4 * L + 3], act, B, h, bn))) return rc;
    return tc_make_map_2d(&host_maps[4 * L + 4], xg2, B, d, bn);
}
