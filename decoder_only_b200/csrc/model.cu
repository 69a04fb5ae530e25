// The model: arena layout, weight initialisation, prefill and decode launch
// sequences, the C ABI of include/llama_b200.h.
//
// Per block ("The one formula"; "Pre-norm: the norm goes on the branch, not
// the trunk"):
//   xn    = RMSNorm(trunk) * g_attn                       rmsnorm kernel
//   Q,K,V = xn [Wq Wk Wv]; RoPE(Q), RoPE(K); K,V -> cache  GEMM + QKV epilogue
//   attn  = causal softmax(Q K^T / sqrt(hd)) V per head     attention kernel
//   trunk += attn Wo                                        GEMM + residual epilogue
//   xn    = RMSNorm(trunk) * g_ffn                          rmsnorm kernel
//   act   = SiLU(xn Wg) * (xn Wu)                           GEMM + SwiGLU epilogue
//   trunk += act Wd                                         GEMM + residual epilogue
// then logits = RMSNorm(trunk) * g_final Whead.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <string>
#include <vector>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

// Programmatic dependent launch on the hot path (LLAMA_B200_NO_PDL=1: off).
bool g_llama_pdl = [] {
    const char* e = getenv("LLAMA_B200_NO_PDL");
    return !(e && e[0] == '1');
}();

// ------------------------------------------------------------------ counters
// Launches of this library's kernels (graph replays count their kernels).
static std::atomic<int64_t> g_launches{0};
void llama_count_launches(int64_t n) { g_launches += n; }

namespace prof {
// Optional per-region timing with CUDA events (eager launches only): each
// region records its device time, its kernel launches and the algorithmic
// bytes / FLOPs it was given.
struct Entry {
    std::string name;
    double ms = 0, bytes = 0, flops = 0;
    int64_t launches = 0, calls = 0;
};
struct Pending {
    int idx;
    cudaEvent_t a, b;
};
static bool on = false;
static std::vector<Entry> entries;
static std::vector<Pending> pending;
static std::vector<cudaEvent_t> pool;

static cudaEvent_t get_event() {
    if (!pool.empty()) {
        cudaEvent_t e = pool.back();
        pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}
static void flush() {
    for (auto& p : pending) {
        float ms = 0.f;
        cudaEventSynchronize(p.b);
        cudaEventElapsedTime(&ms, p.a, p.b);
        entries[p.idx].ms += ms;
        pool.push_back(p.a);
        pool.push_back(p.b);
    }
    pending.clear();
}
static int find(const char* name) {
    for (size_t i = 0; i < entries.size(); ++i)
        if (entries[i].name == name) return (int)i;
    entries.push_back(Entry());
    entries.back().name = name;
    return (int)entries.size() - 1;
}
struct Scope {
    int idx = -1;
    cudaEvent_t a = nullptr;
    cudaStream_t st;
    int64_t l0 = 0;
    Scope(cudaStream_t s, const char* name, double bytes, double flops) : st(s) {
        if (!on) return;
        idx = find(name);
        entries[idx].bytes += bytes;
        entries[idx].flops += flops;
        entries[idx].calls += 1;
        a = get_event();
        cudaEventRecord(a, st);
        l0 = g_launches.load();
    }
    ~Scope() {
        if (idx < 0) return;
        cudaEvent_t b = get_event();
        cudaEventRecord(b, st);
        entries[idx].launches += g_launches.load() - l0;
        pending.push_back({idx, a, b});
        if (pending.size() > 4096) flush();
    }
};
}  // namespace prof

namespace {

constexpr uint32_t TID_EMBED = 1, TID_HEAD = 2;
inline uint32_t layer_tid(int l, int m) { return 16u + 8u * (uint32_t)l + (uint32_t)m; }
// bias variant vectors: bq 0, bk 1, bv 2, bo 3, bg 4, bu 5, bd 6, beta_attn 7, beta_ffn 8
inline uint32_t bias_tid(int l, int k) { return (1u << 20) + 16u * (uint32_t)l + (uint32_t)k; }
constexpr int MAX_COUNTERS = 4096;

struct Layer {
    void *wqkv, *wo, *wgu, *wd;
    float *g_attn, *g_ffn;
    // the bias variant (NULL otherwise), fp32 in weight-row order: Q|K|V, O,
    // gate/up interleaved like W_gu, down; the norm shifts; and the decode
    // step's folded biases b + W beta of the projections that consume a norm
    float *b_qkv = nullptr, *b_o = nullptr, *b_gu = nullptr, *b_d = nullptr;
    float *beta_attn = nullptr, *beta_ffn = nullptr, *c_qkv = nullptr, *c_gu = nullptr;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

// Error word of the standalone ops (the model has its own in its arena).
__device__ int g_op_err_word;
// Work-item counters of the standalone prefill attention op.
__device__ int g_op_attn_sched[2];

// Its device address on the current device: in host code the variable's
// name is only a host-side stand-in, so the address is looked up once per
// device, with that device current.
int op_error_word(int** p) {
    static PerDeviceOnce once;
    static int* addr[LLAMA_MAX_DEVICES];
    int dev = -1;
    LLAMA_CUDA_TRY(cudaGetDevice(&dev));
    int rc = once_per_device(once, [dev]() -> int {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_op_err_word) != cudaSuccess || !a) {
            cudaGetLastError();
            return (int)LLAMA_ERR_CUDA;
        }
        addr[dev] = static_cast<int*>(a);
        return (int)LLAMA_OK;
    });
    if (rc) return rc;
    *p = addr[dev];
    return LLAMA_OK;
}

// The same for the standalone attention op's work-item counters.
int op_attn_sched(int** p) {
    static PerDeviceOnce once;
    static int* addr[LLAMA_MAX_DEVICES];
    int dev = -1;
    LLAMA_CUDA_TRY(cudaGetDevice(&dev));
    int rc = once_per_device(once, [dev]() -> int {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_op_attn_sched) != cudaSuccess || !a) {
            cudaGetLastError();
            return (int)LLAMA_ERR_CUDA;
        }
        addr[dev] = static_cast<int*>(a);
        return (int)LLAMA_OK;
    });
    if (rc) return rc;
    *p = addr[dev];
    return LLAMA_OK;
}

struct llama_model {
    llama_config cfg;
    int esz;                 // bytes per stored element
    uint8_t* arena;
    uint64_t arena_bytes;
    void* embed;
    std::vector<Layer> layers;
    float* g_final;
    void* head;
    float2* rope;
    void* kv;
    size_t kv_layer_elems;   // elements of one of K or V for one layer
    float* trunk;
    void *xn, *q, *attn, *act;
    float* gemm_c;           // fp32 GEMM result for the fp32 path
    float* logits_dec;       // [max_batch, vocab]
    float* partial;          // split-K partials
    size_t partial_elems;
    int* counters;           // split-K arrival counters (zero between launches)
    int* attn_cnt;           // decode-attention arrival counters [max_batch * H]
    CUtensorMap* step_maps;  // decode-step tensor-map table (device) [4L + 5]
    const float** step_gains;  // decode-step gain table (device) [2L + 1]
    const float** step_biases; // decode-step bias table (device) [4L], bias variant only
    unsigned int* step_bar;  // decode-step synchronisation words
    void* step_xg2;          // decode-step FFN-norm input g * x, bf16 [max_batch, d]
    float* step_ssq;         // decode-step block sums of squares [2][64][32]
    float* step_attn_work;   // decode-step attention partials
    unsigned long long* step_timeline;   // decode-step phase stamps (while profiling)
    int2* amax_part;         // greedy-choice chunk results [max_batch][chunks]
    int* amax_cnt;           // and their arrival counters [max_batch]
    float* attn_work;
    uint64_t attn_work_bytes;
    int32_t* tok_cur;        // decode input tokens; argmax writes the next ones here
    int32_t* tok_in;         // prompt tokens copied from the host [max_batch * max_seq]
    int32_t* gen_out;        // generated tokens [max_seq, max_batch]
    float* trunk_last;       // last-position trunk rows [max_batch, d]
    int* d_pos;              // decode position
    int* d_err;              // sticky device error word
    int* attn_sched;         // prefill attention's work-item counters (2 ints, zero between launches)
    int B;                   // batch of the last prefill (0: none)
    int cur_len;             // largest position over the sequences (host)
    std::vector<int> pos_h;  // host mirror of d_pos: each sequence's position (ragged batches)
    int splits_qkv, splits_o, splits_gu, splits_d, splits_head;
    // tensor parallelism (tp > 1): this shard's query heads, key/value heads
    // and FFN hidden units (the full counts when tp == 1), the exchange and
    // its stream, and the events ordering the row blocks between the streams
    int tp, tp_rank, Hl, Hkvl, hl;
    llama_allreduce_fn ar_fn;
    void* ar_ctx;
    int ar_chunks;
    cudaStream_t comm;
    std::vector<cudaEvent_t> tp_ev;   // [3][TP_MAX_CHUNKS]: ready, O exchanged, down exchanged
    // paged KV cache (kv_pages > 0): the page table [max_batch][pps] on the
    // device, whether it holds a valid table, and the positions it covers
    int* pages;
    int pps;
    bool pages_ready;
    int seq_cap;
    cudaStream_t cap_stream;
    cudaGraphExec_t graph;
    int graph_B;
    int64_t graph_kernels;   // kernels per replay of the decode graph
};

namespace {

int hidden_of(const llama_config* c);

// Key/value heads (grouped keys and values); 0 in the config means one per query head
inline int kv_heads(const llama_config* c) { return c->n_kv_heads > 0 ? c->n_kv_heads : c->n_heads; }

// Tensor parallelism: shards, and what one shard holds
constexpr int TP_MAX_CHUNKS = 16;
inline int tp_of(const llama_config* c) { return c->tp_size > 1 ? c->tp_size : 1; }
inline int heads_local(const llama_config* c) { return c->n_heads / tp_of(c); }
inline int kv_local(const llama_config* c) { return kv_heads(c) / tp_of(c); }
inline int hidden_local(const llama_config* c) { return hidden_of(c) / tp_of(c); }

int validate(const llama_config* c) {
    if (!c) return LLAMA_ERR_INVALID_ARG;
    if (c->n_layers < 0 || c->d_model <= 0 || c->n_heads <= 0 || c->vocab <= 0) return LLAMA_ERR_INVALID_ARG;
    if (c->head_dim * c->n_heads != c->d_model) return LLAMA_ERR_INVALID_ARG;
    if (c->n_kv_heads < 0 || c->n_heads % kv_heads(c) != 0) return LLAMA_ERR_INVALID_ARG;
    if (c->dtype != LLAMA_F32 && c->dtype != LLAMA_BF16) return LLAMA_ERR_INVALID_ARG;
    if (c->max_batch <= 0 || c->max_seq <= 0) return LLAMA_ERR_INVALID_ARG;
    if (!(c->norm_eps >= 0.f) || !(c->rope_theta > 0.f)) return LLAMA_ERR_INVALID_ARG;
    if (c->d_model % 32 != 0 || c->d_model > 8192) return LLAMA_ERR_INVALID_ARG;
    if (c->ffn_hidden < 0 || c->ffn_hidden % 128 != 0) return LLAMA_ERR_INVALID_ARG;
    if (c->tp_size < 0 || c->tp_size > 64) return LLAMA_ERR_INVALID_ARG;
    if (c->kv_pages < 0 || (c->kv_pages > 0 && c->dtype != LLAMA_BF16)) return LLAMA_ERR_INVALID_ARG;
    if (c->tp_size > 1) {
        // whole heads, whole key/value heads and whole 128-unit SwiGLU blocks per shard
        const int T = c->tp_size;
        if (c->tp_rank < 0 || c->tp_rank >= T) return LLAMA_ERR_INVALID_ARG;
        if (c->n_heads % T != 0 || kv_heads(c) % T != 0 || hidden_of(c) % (128 * T) != 0)
            return LLAMA_ERR_INVALID_ARG;
    } else if (c->tp_rank != 0) {
        return LLAMA_ERR_INVALID_ARG;
    }
    if (c->dtype == LLAMA_BF16) {
        if (c->head_dim != 64 && c->head_dim != 128) return LLAMA_ERR_INVALID_ARG;
        if (c->d_model % 256 != 0) return LLAMA_ERR_INVALID_ARG;
        if (c->max_batch > 32) return LLAMA_ERR_INVALID_ARG;
        if (c->vocab % 128 != 0) return LLAMA_ERR_INVALID_ARG;   // whole 128-row head tiles
        // arrival counters of the fused decode step: one per 128-row block
        const int64_t qkv_rows = c->d_model + 2 * (int64_t)kv_heads(c) * c->head_dim;
        if (qkv_rows % 128 != 0) return LLAMA_ERR_INVALID_ARG;
        if ((qkv_rows + 3 * (int64_t)c->d_model + hidden_of(c) + c->vocab) / 128 > MAX_COUNTERS)
            return LLAMA_ERR_INVALID_ARG;
    } else {
        if (c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128) return LLAMA_ERR_INVALID_ARG;
    }
    return LLAMA_OK;
}

int hidden_of(const llama_config* c) {
    if (c->ffn_hidden > 0) return c->ffn_hidden;
    const int two_thirds = (8 * c->d_model) / 3;
    return 256 * ((two_thirds + 255) / 256);
}

// Walks the arena layout; with m != NULL assigns the pointers.
uint64_t layout(const llama_config* c, llama_model* m, uint8_t* base) {
    const int esz = c->dtype == LLAMA_BF16 ? 2 : 4;
    // per shard: dq query features, kvd key/value features, h hidden units
    const size_t d = c->d_model, h = hidden_local(c), V = c->vocab, L = c->n_layers;
    const size_t kvd = (size_t)kv_local(c) * c->head_dim;
    const size_t dq = (size_t)heads_local(c) * c->head_dim;
    const size_t nmax = (size_t)c->max_batch * c->max_seq;
    size_t off = 0;
    auto take = [&](size_t bytes) -> void* {
        void* p = base ? base + off : nullptr;
        off += align256(bytes);
        return p;
    };
    void* embed = take(V * d * esz);
    if (m) {
        m->embed = embed;
        m->layers.resize(L);
    }
    for (size_t l = 0; l < L; ++l) {
        Layer ly;
        ly.wqkv = take((dq + 2 * kvd) * d * esz);
        ly.wo = take(d * dq * esz);
        ly.wgu = take(2 * h * d * esz);
        ly.wd = take(d * h * esz);
        ly.g_attn = (float*)take(d * 4);
        ly.g_ffn = (float*)take(d * 4);
        if (c->bias) {
            ly.b_qkv = (float*)take((dq + 2 * kvd) * 4);
            ly.b_o = (float*)take(d * 4);
            ly.b_gu = (float*)take(2 * h * 4);
            ly.b_d = (float*)take(d * 4);
            ly.beta_attn = (float*)take(d * 4);
            ly.beta_ffn = (float*)take(d * 4);
            ly.c_qkv = (float*)take((dq + 2 * kvd) * 4);
            ly.c_gu = (float*)take(2 * h * 4);
        }
        if (m) m->layers[l] = ly;
    }
    float* g_final = (float*)take(d * 4);
    void* head = take(V * d * esz);
    float2* rope = (float2*)take((size_t)c->max_seq * (c->head_dim / 2) * sizeof(float2));
    // KV cache: contiguous [max_batch][n_kv][max_seq][hd] per layer and K / V, or a
    // pool of kv_pages pages [n_kv][KV_PAGE][hd] with a page table [max_batch][pps]
    const size_t pps = ((size_t)c->max_seq + KV_PAGE - 1) / KV_PAGE;
    const size_t kv_layer = c->kv_pages > 0 ? (size_t)c->kv_pages * kv_local(c) * KV_PAGE * c->head_dim
                                            : (size_t)c->max_batch * kv_local(c) * c->max_seq * c->head_dim;
    void* kv = take(2 * L * kv_layer * esz);
    int* pages = (int*)take(c->kv_pages > 0 ? (size_t)c->max_batch * pps * 4 : 0);
    float* trunk = (float*)take(nmax * d * 4);
    void* xn = take(nmax * d * esz);
    void* q = take(nmax * dq * esz);
    void* attn = take(nmax * dq * esz);
    void* act = take(nmax * h * esz);
    const size_t cmax = std::max(dq + 2 * kvd, 2 * h);
    float* gemm_c = (float*)take(c->dtype == LLAMA_F32 ? nmax * std::max(cmax, V) * 4 : 0);
    float* logits_dec = (float*)take((size_t)c->max_batch * V * 4);
    long long part_off[5];
    int cnt_off[5];
    const size_t pmax = (size_t)decode_step_layout(STEP_MAX_CTAS, (int)(d + 2 * kvd), (int)d, (int)h, (int)V,
                                                   c->max_batch, part_off,
                                                   cnt_off);
    float* partial = (float*)take(c->dtype == LLAMA_BF16 ? pmax * 4 : 0);
    int* counters = (int*)take(MAX_COUNTERS * 4);
    int* attn_cnt = (int*)take((size_t)c->max_batch * c->n_heads * 4);
    CUtensorMap* step_maps = (CUtensorMap*)take((size_t)(4 * L + 5) * sizeof(CUtensorMap));
    const float** step_gains = (const float**)take((size_t)(2 * L + 1) * sizeof(float*));
    const float** step_biases = (const float**)take(c->bias ? (size_t)(4 * L) * sizeof(float*) : 0);
    unsigned int* step_bar = (unsigned int*)take(decode_step_sync_words((int)L) * 4);
    void* step_xg2 = take((size_t)c->max_batch * d * esz);
    float* step_ssq = (float*)take(2 * 64 * 32 * 4);
    // attention partials of the fused decode step: pairs * (ranges per pair)
    // <= pairs * (ceil(W / pairs) + 1) <= W + 2 * pairs for W attention warps
    float* step_attn_work = (float*)take(((size_t)STEP_MAX_CTAS * STEP_ATTN_WARPS + 2 * (size_t)c->max_batch *
                                          c->n_heads) * (c->head_dim + 2) * 4);
    // per-phase timestamps of the fused decode step (profiling): 2 per CTA per phase
    unsigned long long* step_timeline = (unsigned long long*)take((size_t)1024 * (3 + 5 * L) * 2 * 8);
    int2* amax_part = (int2*)take((size_t)c->max_batch * argmax_split_chunks(c->vocab) * sizeof(int2));
    int* amax_cnt = (int*)take((size_t)(c->max_batch + 1) * 4);
    const uint64_t awb = attention_decode_work_bytes(c->max_batch, c->n_heads, c->max_seq, c->head_dim);
    float* attn_work = (float*)take(awb);
    int32_t* tok_cur = (int32_t*)take((size_t)c->max_batch * 4);
    int32_t* tok_in = (int32_t*)take(nmax * 4);
    int32_t* gen_out = (int32_t*)take(nmax * 4);
    float* trunk_last = (float*)take((size_t)c->max_batch * d * 4);
    int* small = (int*)take(256);
    int* d_posv = (int*)take((size_t)c->max_batch * 4);
    if (m) {
        m->g_final = g_final;
        m->head = head;
        m->rope = rope;
        m->kv = kv;
        m->kv_layer_elems = kv_layer;
        m->pages = c->kv_pages > 0 ? pages : nullptr;
        m->pps = (int)pps;
        m->trunk = trunk;
        m->xn = xn;
        m->q = q;
        m->attn = attn;
        m->act = act;
        m->gemm_c = gemm_c;
        m->logits_dec = logits_dec;
        m->partial = partial;
        m->partial_elems = pmax;
        m->counters = counters;
        m->amax_part = amax_part;
        m->attn_cnt = attn_cnt;
        m->step_maps = step_maps;
        m->step_gains = step_gains;
        m->step_biases = c->bias ? step_biases : nullptr;
        m->step_bar = step_bar;
        m->step_xg2 = step_xg2;
        m->step_ssq = step_ssq;
        m->step_attn_work = step_attn_work;
        m->step_timeline = step_timeline;
        m->amax_cnt = amax_cnt;
        m->attn_work = attn_work;
        m->attn_work_bytes = awb;
        m->tok_cur = tok_cur;
        m->tok_in = tok_in;
        m->gen_out = gen_out;
        m->trunk_last = trunk_last;
        m->d_pos = d_posv;
        m->d_err = small + 1;
        m->attn_sched = small + 8;
    }
    return off;
}

inline void* kcache(llama_model* m, int l) {
    return (uint8_t*)m->kv + (size_t)(2 * l) * m->kv_layer_elems * m->esz;
}
inline void* vcache(llama_model* m, int l) {
    return (uint8_t*)m->kv + (size_t)(2 * l + 1) * m->kv_layer_elems * m->esz;
}

__global__ void pos_set_kernel(int* pos, int v, int n) {
    pdl_launch_dependents();
    pdl_wait();
    for (int i = threadIdx.x; i < n; i += blockDim.x) pos[i] = v;
}
__global__ void pos_advance_kernel(int* pos, int n) {
    pdl_launch_dependents();
    pdl_wait();
    for (int i = threadIdx.x; i < n; i += blockDim.x) pos[i] += 1;
}
// Logits row of each sequence's last prompt token (position pos[b] - 1) into dst [B, V]
__global__ void last_rows_kernel(const float* logits, const int* pos, int S, int V, float* dst) {
    const int b = blockIdx.y;
    const float* src = logits + ((size_t)b * S + (pos[b] - 1)) * V;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < V; i += gridDim.x * blockDim.x)
        dst[(size_t)b * V + i] = src[i];
}

EpiArgs base_args(llama_model* m, int M, int N) {
    EpiArgs a;
    memset(&a, 0, sizeof(a));
    a.M = M;
    a.N = N;
    a.H = m->Hl;                       // this shard's heads (all of them without tensor parallelism)
    a.Hkv = m->Hkvl;
    a.hd = m->cfg.head_dim;
    a.d = m->Hl * m->cfg.head_dim;     // Q columns of the QKV projection
    a.smax = m->cfg.max_seq;
    a.rope = m->rope;
    a.hidden = m->hl;
    a.pages = m->pages;
    a.pps = m->pps;
    return a;
}

// One projection: out-op(A [M, K] . W [N, K]^T).  mode in EPI_*.
// bf16: tcgen05 GEMM with the fused epilogue (prefill; the bf16 decode step
// is one fused kernel).  fp32: SIMT GEMM + epilogue pass (prefill and
// decode).
double out_bytes(int mode, int M, int N, int esz) {
    switch (mode) {
        case EPI_F32: return (double)M * N * 4;
        case EPI_RESID: return (double)M * N * 8;     // read + write of the fp32 trunk
        case EPI_SWIGLU: return (double)M * (N / 2) * esz;
        default: return (double)M * N * esz;           // Q, K, V
    }
}

int project(llama_model* m, const char* name, int mode, const void* A, const void* W, int M, int N, int K,
            int splits, const EpiArgs& a, bool decode, cudaStream_t st) {
    const int dt = m->cfg.dtype;
    const double esz = m->esz;
    const double flops = 2.0 * M * N * K;
    const double in_bytes = ((double)M * K + (double)N * K) * esz;
    char region[64];
    snprintf(region, sizeof(region), "%s_gemm_%s", decode ? "decode" : "prefill", name);
    if (dt == LLAMA_BF16) {
        TcGemm g;
        if (!decode) {
            prof::Scope ps(st, region, in_bytes + out_bytes(mode, M, N, m->esz), flops);
            g.A = A;
            g.B = W;
            g.rowsA = M;
            g.rowsB = N;
            g.K = K;
            g.splits = 1;
            g.swap = 0;
            return launch_gemm_tc(g, mode, a, m->d_err, st);
        }
        return LLAMA_ERR_INVALID_ARG;   // bf16 decode runs as one fused step (decode_step.cu)
    }
    // fp32 storage: SIMT GEMM
    prof::Scope ps(st, region, in_bytes + out_bytes(mode, M, N, m->esz), flops);
    if (mode == EPI_RESID && !a.bias) return launch_gemm_simt(dt, A, W, a.out, M, N, K, 1, st);
    if (mode == EPI_F32) return launch_gemm_simt(dt, A, W, a.out, M, N, K, 0, st);
    int rc = launch_gemm_simt(dt, A, W, m->gemm_c, M, N, K, 0, st);
    if (rc) return rc;
    return launch_epilogue_from_f32(dt, mode, m->gemm_c, N, a, st);
}

// The L blocks on the trunk [B*S, d] (prefill) or [B, d] (decode).
int run_blocks(llama_model* m, int B, int S, bool decode, cudaStream_t st) {
    const llama_config& c = m->cfg;
    const int d = c.d_model, h = hidden_of(&c);
    const int nq = d + 2 * kv_heads(&c) * c.head_dim;   // Q, K, V columns
    const int Hkv = kv_heads(&c);
    const int n = decode ? B : B * S;
    const int dt = c.dtype;
    int rc;
    for (int l = 0; l < c.n_layers; ++l) {
        const Layer& ly = m->layers[l];
        const double nb = (double)n * d * (4 + m->esz);
        // attention sublayer
        {
            prof::Scope ps(st, decode ? "decode_rmsnorm" : "prefill_rmsnorm", nb, 3.0 * n * d);
            if ((rc = launch_rmsnorm(dt, m->trunk, ly.g_attn, m->xn, n, d, c.norm_eps, st, ly.beta_attn))) return rc;
        }
        EpiArgs qa = base_args(m, n, nq);
        qa.q = m->q;
        qa.kc = kcache(m, l);
        qa.vc = vcache(m, l);
        qa.S = decode ? 1 : S;
        qa.d_pos = decode ? m->d_pos : nullptr;
        qa.bias = ly.b_qkv;
        if ((rc = project(m, "qkv", EPI_QKV, m->xn, ly.wqkv, n, nq, d, m->splits_qkv, qa, decode, st))) return rc;
        if (decode) {
            double len = 0;   // keys read this step, averaged over the sequences
            for (int b = 0; b < B; ++b) len += m->pos_h[b] + 1;
            len /= B;
            prof::Scope ps(st, "decode_attention", (2.0 * len + 2.0) * B * d * m->esz, 4.0 * B * d * len);
            if ((rc = launch_attention_decode(dt, m->q, kcache(m, l), vcache(m, l), m->attn, B, c.n_heads, Hkv, 0,
                                              m->d_pos, c.head_dim, c.max_seq, m->attn_work, m->attn_cnt, m->d_err,
                                              st)))
                return rc;
        } else {
            prof::Scope ps(st, "prefill_attention", 4.0 * n * d * m->esz, 2.0 * B * (double)S * (S + 1) * d);
            if (dt == LLAMA_BF16)
                rc = launch_attention_prefill_tc(m->q, kcache(m, l), vcache(m, l), m->attn, B, c.n_heads, Hkv, S,
                                                 c.head_dim, c.max_seq, m->d_err, m->attn_sched, st, m->pages, m->pps,
                                                 c.kv_pages);
            else
                rc = launch_attention_prefill_simt(dt, m->q, kcache(m, l), vcache(m, l), m->attn, B, c.n_heads, Hkv, S,
                                                   c.head_dim, c.max_seq, st);
            if (rc) return rc;
        }
        EpiArgs ra = base_args(m, n, d);
        ra.out = m->trunk;
        ra.ld_out = d;
        ra.bias = ly.b_o;
        if ((rc = project(m, "o", EPI_RESID, m->attn, ly.wo, n, d, d, m->splits_o, ra, decode, st))) return rc;
        // feed-forward sublayer
        {
            prof::Scope ps(st, decode ? "decode_rmsnorm" : "prefill_rmsnorm", nb, 3.0 * n * d);
            if ((rc = launch_rmsnorm(dt, m->trunk, ly.g_ffn, m->xn, n, d, c.norm_eps, st, ly.beta_ffn))) return rc;
        }
        EpiArgs sa = base_args(m, n, 2 * h);
        sa.act = m->act;
        sa.bias = ly.b_gu;
        ra.bias = ly.b_d;
        if ((rc = project(m, "gateup", EPI_SWIGLU, m->xn, ly.wgu, n, 2 * h, d, m->splits_gu, sa, decode, st))) return rc;
        if ((rc = project(m, "down", EPI_RESID, m->act, ly.wd, n, d, h, m->splits_d, ra, decode, st))) return rc;
    }
    return LLAMA_OK;
}

// ----------------------------------------------------------- tensor parallel
// One projection on token rows [r0, r0 + rows) of A [n, K] (row-major): the
// operand, the outputs and, for the QKV epilogue, the token index of its
// first row move with the block.
int project_rows(llama_model* m, const char* name, int mode, const void* A, const void* W, int r0, int rows,
                 int N, int K, EpiArgs a, cudaStream_t st) {
    const uint8_t* Ar = static_cast<const uint8_t*>(A) + (size_t)r0 * K * m->esz;
    a.M = rows;
    if (a.out) a.out += (size_t)r0 * a.ld_out;
    if (a.act) a.act = static_cast<uint8_t*>(a.act) + (size_t)r0 * a.hidden * m->esz;
    a.m0 = r0;
    return project(m, name, mode, Ar, W, rows, N, K, 1, a, false, st);
}

// The L blocks of a shard ([KN] "Efficient Training Implementation": model
// parallelism with the all-reduce hidden behind computation).  The token
// rows after attention are cut into row blocks; per block, the O (and
// later the down) projection writes this shard's partial into the trunk --
// shard 0 adds it to the trunk and the output bias, the others store it --
// and the exchange sums the block over the shards on the model's own
// stream while the next block computes.  The FFN norm of a block (and, in
// the next layer, the attention norm and QKV projection of a block) waits
// only for that block's exchange.  Attention needs every row of a sequence
// and runs once per layer, between the QKV and O row blocks.
int run_blocks_tp(llama_model* m, int B, int S, cudaStream_t st) {
    const llama_config& c = m->cfg;
    const int d = c.d_model, dq = m->Hl * c.head_dim;
    const int nq = dq + 2 * m->Hkvl * c.head_dim;
    const int n = B * S, dt = c.dtype;
    const int want = std::max(1, std::min(m->ar_chunks, TP_MAX_CHUNKS));
    const int per = std::max(128, ((n + want - 1) / want + 127) / 128 * 128);
    const int nch = (n + per - 1) / per;
    cudaEvent_t* ready = m->tp_ev.data();
    cudaEvent_t* done_o = ready + TP_MAX_CHUNKS;
    cudaEvent_t* done_d = ready + 2 * TP_MAX_CHUNKS;
    const bool lead = m->tp_rank == 0;
    const int out_mode = lead ? EPI_RESID : EPI_F32;
    auto rows_of = [&](int k) { return std::min(per, n - k * per); };
    // queue the sum over the shards of trunk rows of block k after the work queued so far on st
    auto exchange = [&](int k, cudaEvent_t done) -> int {
        LLAMA_CUDA_TRY(cudaEventRecord(ready[k], st));
        LLAMA_CUDA_TRY(cudaStreamWaitEvent(m->comm, ready[k], 0));
        {
            const double bytes = (double)rows_of(k) * d * 4;
            prof::Scope ps(m->comm, "prefill_allreduce", 2.0 * bytes * (m->tp - 1) / m->tp, 0.0);
            if (m->ar_fn(m->trunk + (size_t)k * per * d, (uint64_t)rows_of(k) * d, (void*)m->comm, m->ar_ctx) != 0)
                return LLAMA_ERR_CUDA;
        }
        LLAMA_CUDA_TRY(cudaEventRecord(done, m->comm));
        return LLAMA_OK;
    };
    int rc;
    for (int l = 0; l < c.n_layers; ++l) {
        const Layer& ly = m->layers[l];
        // attention norm + QKV (+ RoPE, KV append) per row block
        for (int k = 0; k < nch; ++k) {
            const int r0 = k * per, rows = rows_of(k);
            if (l > 0) LLAMA_CUDA_TRY(cudaStreamWaitEvent(st, done_d[k], 0));
            {
                prof::Scope ps(st, "prefill_rmsnorm", (double)rows * d * (4 + m->esz), 3.0 * rows * d);
                if ((rc = launch_rmsnorm(dt, m->trunk + (size_t)r0 * d, ly.g_attn,
                                         static_cast<uint8_t*>(m->xn) + (size_t)r0 * d * m->esz, rows, d, c.norm_eps,
                                         st, ly.beta_attn)))
                    return rc;
            }
            EpiArgs qa = base_args(m, rows, nq);
            qa.q = m->q;
            qa.kc = kcache(m, l);
            qa.vc = vcache(m, l);
            qa.S = S;
            qa.bias = ly.b_qkv;
            if ((rc = project_rows(m, "qkv", EPI_QKV, m->xn, ly.wqkv, r0, rows, nq, d, qa, st))) return rc;
        }
        {
            prof::Scope ps(st, "prefill_attention", 4.0 * n * dq * m->esz, 2.0 * B * (double)S * (S + 1) * dq);
            if (dt == LLAMA_BF16)
                rc = launch_attention_prefill_tc(m->q, kcache(m, l), vcache(m, l), m->attn, B, m->Hl, m->Hkvl, S,
                                                 c.head_dim, c.max_seq, m->d_err, m->attn_sched, st, m->pages, m->pps,
                                                 c.kv_pages);
            else
                rc = launch_attention_prefill_simt(dt, m->q, kcache(m, l), vcache(m, l), m->attn, B, m->Hl, m->Hkvl,
                                                   S, c.head_dim, c.max_seq, st);
            if (rc) return rc;
        }
        // O projection: this shard's partial of each row block, then its exchange
        for (int k = 0; k < nch; ++k) {
            EpiArgs ra = base_args(m, rows_of(k), d);
            ra.out = m->trunk;
            ra.ld_out = d;
            ra.bias = lead ? ly.b_o : nullptr;
            if ((rc = project_rows(m, "o", out_mode, m->attn, ly.wo, k * per, rows_of(k), d, dq, ra, st))) return rc;
            if ((rc = exchange(k, done_o[k]))) return rc;
        }
        // FFN per row block, once the block's attention output has been summed
        for (int k = 0; k < nch; ++k) {
            const int r0 = k * per, rows = rows_of(k);
            LLAMA_CUDA_TRY(cudaStreamWaitEvent(st, done_o[k], 0));
            {
                prof::Scope ps(st, "prefill_rmsnorm", (double)rows * d * (4 + m->esz), 3.0 * rows * d);
                if ((rc = launch_rmsnorm(dt, m->trunk + (size_t)r0 * d, ly.g_ffn,
                                         static_cast<uint8_t*>(m->xn) + (size_t)r0 * d * m->esz, rows, d, c.norm_eps,
                                         st, ly.beta_ffn)))
                    return rc;
            }
            EpiArgs sa = base_args(m, rows, 2 * m->hl);
            sa.act = m->act;
            sa.bias = ly.b_gu;
            if ((rc = project_rows(m, "gateup", EPI_SWIGLU, m->xn, ly.wgu, r0, rows, 2 * m->hl, d, sa, st))) return rc;
            EpiArgs ra = base_args(m, rows, d);
            ra.out = m->trunk;
            ra.ld_out = d;
            ra.bias = lead ? ly.b_d : nullptr;
            if ((rc = project_rows(m, "down", out_mode, m->act, ly.wd, r0, rows, d, m->hl, ra, st))) return rc;
            if ((rc = exchange(k, done_d[k]))) return rc;
        }
    }
    for (int k = 0; k < nch; ++k) LLAMA_CUDA_TRY(cudaStreamWaitEvent(st, done_d[k], 0));
    return LLAMA_OK;
}

// The blocks of a prefill: the shard schedule under tensor parallelism.
int prefill_blocks(llama_model* m, int B, int S, cudaStream_t st) {
    if (m->tp > 1) return run_blocks_tp(m, B, S, st);
    return run_blocks(m, B, S, false, st);
}

int run_head(llama_model* m, const float* x, int n, float* logits, bool decode, cudaStream_t st) {
    const llama_config& c = m->cfg;
    int rc;
    {
        prof::Scope ps(st, decode ? "decode_rmsnorm" : "prefill_rmsnorm", (double)n * c.d_model * (4 + m->esz),
                       3.0 * n * c.d_model);
        rc = launch_rmsnorm(c.dtype, x, m->g_final, m->xn, n, c.d_model, c.norm_eps, st);
    }
    if (rc) return rc;
    EpiArgs a = base_args(m, n, c.vocab);
    a.out = logits;
    a.ld_out = c.vocab;
    return project(m, "head", EPI_F32, m->xn, m->head, n, c.vocab, c.d_model, m->splits_head, a, decode, st);
}

// Body of one decode step on the internal buffers: tok_cur -> tok_cur.
// Arguments of the fused bf16 decode step for the current batch.
StepArgs step_args(llama_model* m) {
    const llama_config& c = m->cfg;
    StepArgs a;
    memset(&a, 0, sizeof(a));
    a.maps = m->step_maps;
    a.gains = m->step_gains;
    a.biases = m->step_biases;
    a.embed = (const bf16*)m->embed;
    a.kv = (bf16*)m->kv;
    a.kv_layer = m->kv_layer_elems;
    a.trunk = m->trunk;
    a.xg = (bf16*)m->xn;
    a.xg2 = (bf16*)m->step_xg2;
    a.ssq = m->step_ssq;
    a.q = (bf16*)m->q;
    a.attn = (bf16*)m->attn;
    a.act = (bf16*)m->act;
    a.logits = m->logits_dec;
    a.partial = m->partial;
    a.counters = m->counters;
    decode_step_layout(decode_step_ctas(), c.d_model + 2 * kv_heads(&c) * c.head_dim, c.d_model, c.ffn_hidden,
                       c.vocab, m->B, a.part_off, a.cnt_off);
    a.attn_work = m->step_attn_work;
    a.attn_cnt = m->attn_cnt;
    a.amax_part = m->amax_part;
    a.amax_cnt = m->amax_cnt;
    a.tok = m->tok_cur;
    a.d_pos = m->d_pos;
    a.err = m->d_err;
    a.bar = m->step_bar;
    a.rope = m->rope;
    a.L = c.n_layers;
    a.d = c.d_model;
    a.h = c.ffn_hidden;
    a.V = c.vocab;
    a.H = c.n_heads;
    a.Hkv = kv_heads(&c);
    a.hd = c.head_dim;
    a.B = m->B;
    a.smax = c.max_seq;
    a.eps = c.norm_eps;
    a.pages = m->pages;
    a.pps = m->pps;
    return a;
}

// Tensor maps and gain pointers of the fused decode step (synchronous copy
// into the arena; done before the step graph is captured).
int step_tables(llama_model* m) {
    const llama_config& c = m->cfg;
    const int L = c.n_layers;
    std::vector<CUtensorMap> maps((size_t)4 * L + 5);
    std::vector<const void*> w((size_t)4 * L);
    for (int l = 0; l < L; ++l) {
        w[4 * l + 0] = m->layers[l].wqkv;
        w[4 * l + 1] = m->layers[l].wo;
        w[4 * l + 2] = m->layers[l].wgu;
        w[4 * l + 3] = m->layers[l].wd;
    }
    int rc = decode_step_maps(maps.data(), w.data(), L, m->head, m->xn, m->attn, m->act, m->step_xg2, m->B,
                              c.d_model + 2 * kv_heads(&c) * c.head_dim,
                              c.d_model, c.ffn_hidden, c.vocab);
    if (rc) return rc;
    std::vector<const float*> gains((size_t)2 * L + 1);
    for (int l = 0; l < L; ++l) {
        gains[2 * l] = m->layers[l].g_attn;
        gains[2 * l + 1] = m->layers[l].g_ffn;
    }
    gains[2 * L] = m->g_final;
    LLAMA_CUDA_TRY(cudaMemcpy(m->step_maps, maps.data(), maps.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice));
    LLAMA_CUDA_TRY(cudaMemcpy(m->step_gains, gains.data(), gains.size() * sizeof(float*), cudaMemcpyHostToDevice));
    if (m->step_biases) {
        std::vector<const float*> bt((size_t)4 * L);
        for (int l = 0; l < L; ++l) {
            bt[4 * l + 0] = m->layers[l].c_qkv;
            bt[4 * l + 1] = m->layers[l].b_o;
            bt[4 * l + 2] = m->layers[l].c_gu;
            bt[4 * l + 3] = m->layers[l].b_d;
        }
        LLAMA_CUDA_TRY(cudaMemcpy(m->step_biases, bt.data(), bt.size() * sizeof(float*), cudaMemcpyHostToDevice));
    }
    return LLAMA_OK;
}

int decode_body(llama_model* m, cudaStream_t st) {
    const llama_config& c = m->cfg;
    int rc;
    if (c.dtype == LLAMA_BF16) {
        // weights + KV cache read + activations, once per step
        const double d = c.d_model, h = c.ffn_hidden, L = c.n_layers, V = c.vocab;
        const double kvd = (double)kv_heads(&c) * c.head_dim;
        const double wbytes = 2.0 * (L * (2 * d * d + 2 * d * kvd + 3 * d * h) + d * V);
        double keys = 0;   // keys read this step, over the sequences
        for (int b = 0; b < m->B; ++b) keys += m->pos_h[b] + 1;
        const double kvbytes = 2.0 * 2.0 * L * keys * kvd;
        const double flops = 2.0 * m->B * (L * (2 * d * d + 2 * d * kvd + 3 * d * h) + d * V) + 4.0 * L * keys * d;
        prof::Scope ps(st, "decode_step", wbytes + kvbytes, flops);
        StepArgs sa = step_args(m);
        if (prof::on) sa.timeline = m->step_timeline;
        return launch_decode_step(sa, st);
    }
    {
        prof::Scope ps(st, "decode_embed", (double)m->B * c.d_model * (4 + m->esz), 0.0);
        rc = launch_embed(c.dtype, m->tok_cur, m->embed, m->trunk, m->B, c.d_model, c.vocab, m->d_err, st);
    }
    if (rc) return rc;
    if ((rc = run_blocks(m, m->B, 1, true, st))) return rc;
    if ((rc = run_head(m, m->trunk, m->B, m->logits_dec, true, st))) return rc;
    prof::Scope ps(st, "decode_argmax", (double)m->B * c.vocab * 4, 0.0);
    if ((rc = launch_argmax_split(m->logits_dec, m->B, c.vocab, c.vocab, m->tok_cur, m->amax_part, m->amax_cnt, st)))
        return rc;
    launch_pdl(pos_advance_kernel, dim3(1), dim3(32), 0, st, m->d_pos, m->B);
    LLAMA_LAUNCH_CHECK();
    return LLAMA_OK;
}

// One decode step: the captured graph, or eager launches while profiling.
int decode_once(llama_model* m, cudaStream_t st) {
    if (prof::on) return decode_body(m, st);
    LLAMA_CUDA_TRY(cudaGraphLaunch(m->graph, st));
    llama_count_launches(m->graph_kernels);
    return LLAMA_OK;
}

int ensure_graph(llama_model* m) {
    if (m->graph && m->graph_B == m->B) return LLAMA_OK;
    if (m->cfg.dtype == LLAMA_BF16) {
        int rc = step_tables(m);
        if (rc) return rc;
    }
    if (m->graph) {
        cudaGraphExecDestroy(m->graph);
        m->graph = nullptr;
    }
    cudaGraph_t g = nullptr;
    const bool prof_was = prof::on;
    prof::on = false;
    const int64_t l0 = g_launches.load();
    LLAMA_CUDA_TRY(cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal));
    int rc = decode_body(m, m->cap_stream);
    cudaError_t e = cudaStreamEndCapture(m->cap_stream, &g);
    prof::on = prof_was;
    m->graph_kernels = g_launches.load() - l0;   // captured, not run
    g_launches -= m->graph_kernels;
    if (rc) {
        if (g) cudaGraphDestroy(g);
        return rc;
    }
    if (e != cudaSuccess) return LLAMA_ERR_CUDA;
    e = cudaGraphInstantiate(&m->graph, g, 0);
    cudaGraphDestroy(g);
    if (e != cudaSuccess) {
        m->graph = nullptr;
        return LLAMA_ERR_CUDA;
    }
    m->graph_B = m->B;
    return LLAMA_OK;
}

void pick_decode_splits(llama_model* m) {
    const llama_config& c = m->cfg;
    const int d = c.d_model, h = hidden_of(&c);
    if (c.dtype != LLAMA_BF16) {
        m->splits_qkv = m->splits_o = m->splits_gu = m->splits_d = m->splits_head = 1;
        return;
    }
    m->splits_qkv = gemm_tc_pick_splits(d + 2 * kv_heads(&c) * c.head_dim, d);
    m->splits_o = gemm_tc_pick_splits(d, d);
    m->splits_gu = gemm_tc_pick_splits(2 * h, d);
    m->splits_d = gemm_tc_pick_splits(d, h);
    m->splits_head = gemm_tc_pick_splits(c.vocab, d);
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

const char* llama_status_str(int s) {
    switch (s) {
        case LLAMA_OK: return "ok";
        case LLAMA_ERR_INVALID_ARG: return "invalid argument";
        case LLAMA_ERR_OOM: return "arena or workspace too small";
        case LLAMA_ERR_CUDA: return "CUDA error";
        case LLAMA_ERR_TIMEOUT: return "bounded device wait expired";
        case LLAMA_ERR_STATE: return "call out of order";
        default: return "unknown status";
    }
}

int llama_model_bytes(const llama_config* cfg, uint64_t* bytes_out) {
    int rc = validate(cfg);
    if (rc) return rc;
    if (!bytes_out) return LLAMA_ERR_INVALID_ARG;
    *bytes_out = layout(cfg, nullptr, nullptr);
    return LLAMA_OK;
}

int llama_init_weights(const llama_config* cfg, uint32_t seed, void* d_arena, uint64_t arena_bytes, void* stream,
                       llama_model** out) {
    int rc = validate(cfg);
    if (rc) return rc;
    if (!out || !d_arena || (reinterpret_cast<uintptr_t>(d_arena) & 255u)) return LLAMA_ERR_INVALID_ARG;
    const uint64_t need = layout(cfg, nullptr, nullptr);
    if (arena_bytes < need) return LLAMA_ERR_OOM;
    cudaStream_t st = (cudaStream_t)stream;
    llama_model* m = new llama_model();
    m->cfg = *cfg;
    m->cfg.ffn_hidden = hidden_of(cfg);
    m->esz = cfg->dtype == LLAMA_BF16 ? 2 : 4;
    m->arena = (uint8_t*)d_arena;
    m->arena_bytes = arena_bytes;
    layout(&m->cfg, m, m->arena);
    m->B = 0;
    m->cur_len = 0;
    m->graph = nullptr;
    m->graph_B = 0;
    m->graph_kernels = 0;
    m->tp = tp_of(cfg);
    m->tp_rank = m->tp > 1 ? cfg->tp_rank : 0;
    m->Hl = heads_local(cfg);
    m->Hkvl = kv_local(cfg);
    m->hl = hidden_local(cfg);
    m->ar_fn = nullptr;
    m->ar_ctx = nullptr;
    m->ar_chunks = 1;
    m->comm = nullptr;
    m->cap_stream = nullptr;
    m->pages_ready = m->pages == nullptr;
    m->seq_cap = cfg->max_seq;
    if (cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking) != cudaSuccess) {
        delete m;
        return LLAMA_ERR_CUDA;
    }
    if (m->tp > 1) {
        bool ok = cudaStreamCreateWithFlags(&m->comm, cudaStreamNonBlocking) == cudaSuccess;
        m->tp_ev.assign(3 * TP_MAX_CHUNKS, nullptr);
        for (auto& e : m->tp_ev) ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
        if (!ok) {
            llama_free(m);
            return LLAMA_ERR_CUDA;
        }
    }
    const int dt = cfg->dtype;
    const int d = cfg->d_model, h = m->cfg.ffn_hidden, V = cfg->vocab;
    const double sc = 0.02;
#define TRY(x)                  \
    do {                        \
        if ((rc = (x))) {       \
            llama_free(m);      \
            return rc;          \
        }                       \
    } while (0)
    TRY(launch_init_matrix(dt, m->embed, d, V, V, 0, 0, 1, seed, TID_EMBED, sc, st));
    TRY(launch_init_matrix(dt, m->head, d, V, V, 0, 0, 0, seed, TID_HEAD, sc, st));
    TRY(launch_fill_f32(m->g_final, 1.0f, d, st));
    // A shard holds slices of the full matrices: query / key / value
    // columns of its heads, the matching input rows of Wo, and the gate / up
    // columns and Wdown input rows of its hidden units (r = 0, T = 1: all).
    const int r = m->tp_rank;
    const int kvd = kv_heads(cfg) * cfg->head_dim;        // full key/value width
    const int dql = m->Hl * cfg->head_dim;                // this shard's query, key/value and hidden widths
    const int kvl = m->Hkvl * cfg->head_dim;
    const int hl = m->hl;
    for (int l = 0; l < cfg->n_layers; ++l) {
        const Layer& ly = m->layers[l];
        // W_qkv rows: the shard's Q columns, then its K, then its V
        TRY(launch_init_shard(dt, ly.wqkv, d, d, 0, d, r * dql, dql, dql, 0, 0, 0, seed, layer_tid(l, 0), sc, st));
        TRY(launch_init_shard(dt, ly.wqkv, d, kvd, 0, d, r * kvl, kvl, kvl, 0, dql, 0, seed, layer_tid(l, 1), sc,
                              st));
        TRY(launch_init_shard(dt, ly.wqkv, d, kvd, 0, d, r * kvl, kvl, kvl, 0, dql + kvl, 0, seed, layer_tid(l, 2),
                              sc, st));
        TRY(launch_init_shard(dt, ly.wo, d, d, r * dql, dql, 0, d, d, 0, 0, 0, seed, layer_tid(l, 3), sc, st));
        TRY(launch_init_shard(dt, ly.wgu, d, h, 0, d, r * hl, hl, 128, 256, 0, 0, seed, layer_tid(l, 4), sc, st));
        TRY(launch_init_shard(dt, ly.wgu, d, h, 0, d, r * hl, hl, 128, 256, 128, 0, seed, layer_tid(l, 5), sc, st));
        TRY(launch_init_shard(dt, ly.wd, h, d, r * hl, hl, 0, d, d, 0, 0, 0, seed, layer_tid(l, 6), sc, st));
        TRY(launch_fill_f32(ly.g_attn, 1.0f, d, st));
        TRY(launch_fill_f32(ly.g_ffn, 1.0f, d, st));
        if (cfg->bias) {
            // vectors of the bias variant: the generator with K = 1 (element j of
            // the vector); a shard holds the slice of the biases of its columns
            auto vec = [&](float* dst, int n_full, int n0, int n_loc, int blk, int blk_stride, int row_off, int k) {
                return launch_init_shard(LLAMA_F32, dst, 1, n_full, 0, 1, n0, n_loc, blk, blk_stride, row_off, 0, seed,
                                         bias_tid(l, k), sc, st);
            };
            TRY(vec(ly.b_qkv, d, r * dql, dql, dql, 0, 0, 0));
            TRY(vec(ly.b_qkv, kvd, r * kvl, kvl, kvl, 0, dql, 1));
            TRY(vec(ly.b_qkv, kvd, r * kvl, kvl, kvl, 0, dql + kvl, 2));
            TRY(vec(ly.b_o, d, 0, d, d, 0, 0, 3));
            TRY(vec(ly.b_gu, h, r * hl, hl, 128, 256, 0, 4));
            TRY(vec(ly.b_gu, h, r * hl, hl, 128, 256, 128, 5));
            TRY(vec(ly.b_d, d, 0, d, d, 0, 0, 6));
            TRY(vec(ly.beta_attn, d, 0, d, d, 0, 0, 7));
            TRY(vec(ly.beta_ffn, d, 0, d, d, 0, 0, 8));
            // decode step: W (g x / rms + beta) + b = W (g x) / rms + (b + W beta)
            TRY(launch_bias_fold(dt, ly.wqkv, dql + 2 * kvl, d, ly.beta_attn, ly.b_qkv, ly.c_qkv, st));
            TRY(launch_bias_fold(dt, ly.wgu, 2 * hl, d, ly.beta_ffn, ly.b_gu, ly.c_gu, st));
        }
    }
    // RoPE table: angle = pos * theta^(-2i/hd), cos and sin in fp64, stored fp32
    const int hp = cfg->head_dim / 2;
    std::vector<float2> tab((size_t)cfg->max_seq * hp);
    for (int p = 0; p < cfg->max_seq; ++p)
        for (int i = 0; i < hp; ++i) {
            const double ang = (double)p * pow((double)cfg->rope_theta, -(2.0 * i) / (double)cfg->head_dim);
            tab[(size_t)p * hp + i] = make_float2((float)cos(ang), (float)sin(ang));
        }
    if (cudaMemcpyAsync(m->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice, st) !=
        cudaSuccess) {
        llama_free(m);
        return LLAMA_ERR_CUDA;
    }
    if (cudaMemsetAsync(m->counters, 0, MAX_COUNTERS * 4, st) != cudaSuccess ||
        cudaMemsetAsync(m->amax_cnt, 0, (size_t)(cfg->max_batch + 1) * 4, st) != cudaSuccess ||
        cudaMemsetAsync(m->step_bar, 0, decode_step_sync_words(cfg->n_layers) * 4, st) != cudaSuccess ||
        cudaMemsetAsync(m->attn_cnt, 0, (size_t)cfg->max_batch * cfg->n_heads * 4, st) != cudaSuccess ||
        cudaMemsetAsync(m->d_pos, 0, (size_t)cfg->max_batch * 4, st) != cudaSuccess ||
        cudaMemsetAsync(m->d_err - 1, 0, 256, st) != cudaSuccess) {
        llama_free(m);
        return LLAMA_ERR_CUDA;
    }
    if (m->pages) {
        // pages start zeroed (a page's rows past its sequence's length are read, masked,
        // by the prefill attention: they must be finite); the default table gives
        // sequence b pages b * pps .. when the pool holds that many
        if (cudaMemsetAsync(m->kv, 0, 2 * (size_t)cfg->n_layers * m->kv_layer_elems * m->esz, st) != cudaSuccess) {
            llama_free(m);
            return LLAMA_ERR_CUDA;
        }
        if ((int64_t)cfg->kv_pages >= (int64_t)cfg->max_batch * m->pps) {
            std::vector<int> tab((size_t)cfg->max_batch * m->pps);
            for (size_t i = 0; i < tab.size(); ++i) tab[i] = (int)i;
            if (cudaMemcpyAsync(m->pages, tab.data(), tab.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess ||
                cudaStreamSynchronize(st) != cudaSuccess) {
                llama_free(m);
                return LLAMA_ERR_CUDA;
            }
            m->pages_ready = true;
        } else {
            m->seq_cap = 0;   // positions need pages: llama_set_pages first
        }
    }
    pick_decode_splits(m);
    if ((rc = gemm_tc_prepare()) || (rc = attention_prepare()) || (rc = attention_tc_prepare()) ||
        (rc = attention_decode_prepare()) || (cfg->dtype == LLAMA_BF16 && (rc = decode_step_prepare()))) {
        llama_free(m);
        return rc;
    }
    if (cudaStreamSynchronize(st) != cudaSuccess) {
        llama_free(m);
        return LLAMA_ERR_CUDA;
    }
#undef TRY
    *out = m;
    return LLAMA_OK;
}

// Prefill of B sequences given as a [B, S] token block; with h_lens
// sequence b holds only its first h_lens[b] tokens (the rest are padding
// with valid ids, whose rows are computed and ignored: causality keeps
// them out of every valid row) and continues at position h_lens[b].
static int prefill_impl(llama_model* m, const int32_t* d_tokens, int32_t B, int32_t S, const int32_t* h_lens,
                        float* d_logits, cudaStream_t st) {
    if (!m || !d_tokens || B <= 0 || S <= 0 || B > m->cfg.max_batch || S > m->cfg.max_seq)
        return LLAMA_ERR_INVALID_ARG;
    if (h_lens)
        for (int b = 0; b < B; ++b)
            if (h_lens[b] < 1 || h_lens[b] > S) return LLAMA_ERR_INVALID_ARG;
    if (m->tp > 1 && !m->ar_fn) return LLAMA_ERR_STATE;   // a shard needs its exchange
    if (!m->pages_ready) return LLAMA_ERR_STATE;         // a paged cache needs its page table
    if (S > m->seq_cap) return LLAMA_ERR_INVALID_ARG;    // positions beyond the sequences' pages
    const int n = B * S;
    const int V = m->cfg.vocab;
    int rc;
    {
        prof::Scope ps(st, "prefill_embed", (double)n * m->cfg.d_model * (4 + m->esz), 0.0);
        rc = launch_embed(m->cfg.dtype, d_tokens, m->embed, m->trunk, n, m->cfg.d_model, V, m->d_err, st);
    }
    if (rc) return rc;
    if ((rc = prefill_blocks(m, B, S, st))) return rc;
    // positions: where each sequence continues
    if (h_lens) {
        LLAMA_CUDA_TRY(cudaMemcpyAsync(m->d_pos, h_lens, (size_t)B * 4, cudaMemcpyHostToDevice, st));
    } else {
        launch_pdl(pos_set_kernel, dim3(1), dim3(32), 0, st, m->d_pos, (int)S, (int)B);
        LLAMA_LAUNCH_CHECK();
    }
    if (d_logits) {
        if ((rc = run_head(m, m->trunk, n, d_logits, false, st))) return rc;
        // greedy choice at each sequence's last prompt token: the input of the
        // first decode step when llama_generate is given no tokens
        prof::Scope ps(st, "prefill_argmax", (double)B * V * 4, 0.0);
        if (h_lens) {
            last_rows_kernel<<<dim3((V + 1023) / 1024, B), 256, 0, st>>>(d_logits, m->d_pos, S, V, m->logits_dec);
            LLAMA_LAUNCH_CHECK();
            rc = launch_argmax_split(m->logits_dec, B, V, V, m->tok_cur, m->amax_part, m->amax_cnt, st);
        } else {
            rc = launch_argmax_split(d_logits + (size_t)(S - 1) * V, B, V, (int64_t)S * V, m->tok_cur, m->amax_part,
                                     m->amax_cnt, st);
        }
        if (rc) return rc;
    }
    m->B = B;
    m->pos_h.assign(B, S);
    if (h_lens) m->pos_h.assign(h_lens, h_lens + B);
    m->cur_len = 0;
    for (int b = 0; b < B; ++b) m->cur_len = std::max(m->cur_len, m->pos_h[b]);
    return LLAMA_OK;
}

int llama_prefill(llama_model* m, const int32_t* d_tokens, int32_t B, int32_t S, float* d_logits, void* stream) {
    return prefill_impl(m, d_tokens, B, S, nullptr, d_logits, (cudaStream_t)stream);
}

int llama_prefill_ragged(llama_model* m, const int32_t* d_tokens, int32_t B, int32_t S, const int32_t* h_lens,
                         float* d_logits, void* stream) {
    if (!h_lens) return LLAMA_ERR_INVALID_ARG;
    return prefill_impl(m, d_tokens, B, S, h_lens, d_logits, (cudaStream_t)stream);
}

int llama_prefill_trunk(llama_model* m, const float* d_x, int32_t B, int32_t S, float* d_y, void* stream) {
    if (!m || !d_x || !d_y || B <= 0 || S <= 0 || B > m->cfg.max_batch || S > m->cfg.max_seq)
        return LLAMA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t bytes = (size_t)B * S * m->cfg.d_model * 4;
    if (m->tp > 1 && !m->ar_fn) return LLAMA_ERR_STATE;
    if (!m->pages_ready) return LLAMA_ERR_STATE;
    if (S > m->seq_cap) return LLAMA_ERR_INVALID_ARG;
    if (d_x != m->trunk) LLAMA_CUDA_TRY(cudaMemcpyAsync(m->trunk, d_x, bytes, cudaMemcpyDeviceToDevice, st));
    int rc = prefill_blocks(m, B, S, st);
    if (rc) return rc;
    if (d_y != m->trunk) LLAMA_CUDA_TRY(cudaMemcpyAsync(d_y, m->trunk, bytes, cudaMemcpyDeviceToDevice, st));
    launch_pdl(pos_set_kernel, dim3(1), dim3(32), 0, st, m->d_pos, (int)S, (int)B);
    LLAMA_LAUNCH_CHECK();
    m->B = B;
    m->cur_len = S;
    m->pos_h.assign(B, S);
    return LLAMA_OK;
}

int llama_decode_step(llama_model* m, const int32_t* d_tokens, int32_t* d_next, float* d_logits, void* stream) {
    if (!m || !d_tokens || m->tp > 1) return LLAMA_ERR_INVALID_ARG;
    if (m->B <= 0 || m->cur_len >= m->cfg.max_seq || m->cur_len >= m->seq_cap) return LLAMA_ERR_STATE;
    cudaStream_t st = (cudaStream_t)stream;
    int rc = ensure_graph(m);
    if (rc) return rc;
    LLAMA_CUDA_TRY(cudaMemcpyAsync(m->tok_cur, d_tokens, (size_t)m->B * 4, cudaMemcpyDeviceToDevice, st));
    if ((rc = decode_once(m, st))) return rc;
    if (d_next) LLAMA_CUDA_TRY(cudaMemcpyAsync(d_next, m->tok_cur, (size_t)m->B * 4, cudaMemcpyDeviceToDevice, st));
    if (d_logits)
        LLAMA_CUDA_TRY(cudaMemcpyAsync(d_logits, m->logits_dec, (size_t)m->B * m->cfg.vocab * 4,
                                       cudaMemcpyDeviceToDevice, st));
    m->cur_len += 1;
    for (int& p : m->pos_h) p += 1;
    return LLAMA_OK;
}

int llama_generate(llama_model* m, const int32_t* d_first, int32_t n_steps, int32_t* d_out, void* stream) {
    if (!m || !d_out || n_steps < 0 || m->tp > 1) return LLAMA_ERR_INVALID_ARG;
    if (m->B <= 0 || m->cur_len + n_steps > m->cfg.max_seq || m->cur_len + n_steps > m->seq_cap)
        return LLAMA_ERR_STATE;
    cudaStream_t st = (cudaStream_t)stream;
    int rc = ensure_graph(m);
    if (rc) return rc;
    if (d_first)
        LLAMA_CUDA_TRY(cudaMemcpyAsync(m->tok_cur, d_first, (size_t)m->B * 4, cudaMemcpyDeviceToDevice, st));
    for (int i = 0; i < n_steps; ++i) {
        if ((rc = decode_once(m, st))) return rc;
        LLAMA_CUDA_TRY(cudaMemcpyAsync(d_out + (size_t)i * m->B, m->tok_cur, (size_t)m->B * 4,
                                       cudaMemcpyDeviceToDevice, st));
        m->cur_len += 1;
        for (int& p : m->pos_h) p += 1;
    }
    return LLAMA_OK;
}

int llama_set_allreduce(llama_model* m, llama_allreduce_fn fn, void* ctx, int32_t chunks) {
    if (!m || !fn || chunks < 1 || chunks > TP_MAX_CHUNKS || m->tp <= 1) return LLAMA_ERR_INVALID_ARG;
    m->ar_fn = fn;
    m->ar_ctx = ctx;
    m->ar_chunks = chunks;
    return LLAMA_OK;
}

int llama_set_pages(llama_model* m, const int32_t* h_table, int32_t B, int32_t pages_per_seq, void* stream) {
    if (!m || !m->pages || !h_table || B < 1 || B > m->cfg.max_batch || pages_per_seq < 1 ||
        pages_per_seq > m->pps)
        return LLAMA_ERR_INVALID_ARG;
    // every page in range, and no page given to two (sequence, position) slots
    std::vector<int> tab((size_t)m->cfg.max_batch * m->pps, 0);
    std::vector<char> used((size_t)m->cfg.kv_pages, 0);
    for (int b = 0; b < B; ++b)
        for (int p = 0; p < pages_per_seq; ++p) {
            const int pg = h_table[(size_t)b * pages_per_seq + p];
            if (pg < 0 || pg >= m->cfg.kv_pages || used[pg]) return LLAMA_ERR_INVALID_ARG;
            used[pg] = 1;
            tab[(size_t)b * m->pps + p] = pg;
        }
    cudaStream_t st = (cudaStream_t)stream;
    LLAMA_CUDA_TRY(cudaMemcpyAsync(m->pages, tab.data(), tab.size() * 4, cudaMemcpyHostToDevice, st));
    LLAMA_CUDA_TRY(cudaStreamSynchronize(st));   // the host table is the caller's again on return
    m->pages_ready = true;
    m->seq_cap = std::min(m->cfg.max_seq, pages_per_seq * KV_PAGE);
    return LLAMA_OK;
}

int llama_tp_shard(const llama_config* cfg, int32_t* h_out) {
    int rc = validate(cfg);
    if (rc) return rc;
    if (!h_out) return LLAMA_ERR_INVALID_ARG;
    const int r = tp_of(cfg) > 1 ? cfg->tp_rank : 0;
    h_out[0] = r * heads_local(cfg);
    h_out[1] = heads_local(cfg);
    h_out[2] = r * kv_local(cfg);
    h_out[3] = kv_local(cfg);
    h_out[4] = r * hidden_local(cfg);
    h_out[5] = hidden_local(cfg);
    return LLAMA_OK;
}

int llama_position(const llama_model* m) { return m ? m->cur_len : LLAMA_ERR_INVALID_ARG; }

int llama_positions(const llama_model* m, int32_t* h_out, int32_t n) {
    if (!m || !h_out || n < m->B) return LLAMA_ERR_INVALID_ARG;
    for (int b = 0; b < m->B; ++b) h_out[b] = m->pos_h[b];
    return m->B;
}

int llama_rewind(llama_model* m, int32_t position, void* stream) {
    if (!m || position < 1) return LLAMA_ERR_INVALID_ARG;
    if (m->B <= 0) return LLAMA_ERR_STATE;
    for (int b = 0; b < m->B; ++b)
        if (position > m->pos_h[b]) return LLAMA_ERR_INVALID_ARG;   // every sequence holds `position` keys
    launch_pdl(pos_set_kernel, dim3(1), dim3(32), 0, (cudaStream_t)stream, m->d_pos, (int)position, m->B);
    LLAMA_LAUNCH_CHECK();
    m->cur_len = position;
    m->pos_h.assign(m->B, position);
    return LLAMA_OK;
}

int llama_complete(llama_model* m, const int32_t* h_tokens, int32_t B, int32_t S, float* d_logits, int32_t n_steps,
                   int32_t* h_out, void* stream) {
    if (!m || !h_tokens || !h_out || B <= 0 || S <= 0 || n_steps < 0 || B > m->cfg.max_batch ||
        S + n_steps > m->cfg.max_seq || m->tp > 1)
        return LLAMA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const llama_config& c = m->cfg;
    LLAMA_CUDA_TRY(cudaMemcpyAsync(m->tok_in, h_tokens, (size_t)B * S * 4, cudaMemcpyHostToDevice, st));
    int rc = llama_prefill(m, m->tok_in, B, S, d_logits, stream);
    if (rc) return rc;
    if (!d_logits) {
        // head on the last position of each sequence only
        LLAMA_CUDA_TRY(cudaMemcpy2DAsync(m->trunk_last, (size_t)c.d_model * 4, m->trunk + (size_t)(S - 1) * c.d_model,
                                         (size_t)S * c.d_model * 4, (size_t)c.d_model * 4, B,
                                         cudaMemcpyDeviceToDevice, st));
        if ((rc = run_head(m, m->trunk_last, B, m->logits_dec, true, st))) return rc;
        if ((rc = launch_argmax_split(m->logits_dec, B, c.vocab, c.vocab, m->tok_cur, m->amax_part, m->amax_cnt,
                                      st)))
            return rc;
    }
    if ((rc = llama_generate(m, nullptr, n_steps, m->gen_out, stream))) return rc;
    LLAMA_CUDA_TRY(cudaMemcpyAsync(h_out, m->gen_out, (size_t)n_steps * B * 4, cudaMemcpyDeviceToHost, st));
    return LLAMA_OK;
}

int llama_model_tensor(const llama_model* m, const char* name, int32_t layer, void** d_ptr, uint64_t* bytes) {
    if (!m || !name || !d_ptr || !bytes) return LLAMA_ERR_INVALID_ARG;
    const llama_config& c = m->cfg;
    const size_t d = c.d_model, h = m->hl, V = c.vocab, es = m->esz;   // h, dq: this shard's widths
    const size_t dq = (size_t)m->Hl * c.head_dim;
    const size_t nmax = (size_t)c.max_batch * c.max_seq;
    auto lay = [&](int l) -> const Layer* { return (l >= 0 && l < c.n_layers) ? &m->layers[l] : nullptr; };
    if (!strcmp(name, "kv")) { *d_ptr = m->kv; *bytes = 2 * (size_t)c.n_layers * m->kv_layer_elems * es; }
    else if (!strcmp(name, "trunk")) { *d_ptr = m->trunk; *bytes = nmax * d * 4; }
    else if (!strcmp(name, "q")) { *d_ptr = m->q; *bytes = nmax * dq * es; }
    else if (!strcmp(name, "attn")) { *d_ptr = m->attn; *bytes = nmax * dq * es; }
    else if (!strcmp(name, "xn")) { *d_ptr = m->xn; *bytes = nmax * d * es; }
    else if (!strcmp(name, "act")) { *d_ptr = m->act; *bytes = nmax * h * es; }
    else if (!strcmp(name, "embed")) { *d_ptr = m->embed; *bytes = V * d * es; }
    else if (!strcmp(name, "head")) { *d_ptr = m->head; *bytes = V * d * es; }
    else if (!strcmp(name, "logits_dec")) { *d_ptr = m->logits_dec; *bytes = (size_t)c.max_batch * V * 4; }
    else {
        const Layer* ly = lay(layer);
        if (!ly) return LLAMA_ERR_INVALID_ARG;
        if (!strcmp(name, "wqkv")) {
            *d_ptr = ly->wqkv;
            *bytes = (dq + 2 * (size_t)m->Hkvl * c.head_dim) * d * es;
        }
        else if (!strcmp(name, "wo")) { *d_ptr = ly->wo; *bytes = d * dq * es; }
        else if (!strcmp(name, "wgu")) { *d_ptr = ly->wgu; *bytes = 2 * h * d * es; }
        else if (!strcmp(name, "wd")) { *d_ptr = ly->wd; *bytes = d * h * es; }
        else return LLAMA_ERR_INVALID_ARG;
    }
    return LLAMA_OK;
}

int llama_last_error(llama_model* m) {
    if (!m) return LLAMA_ERR_INVALID_ARG;
    int e = 0;
    LLAMA_CUDA_TRY(cudaMemcpy(&e, m->d_err, sizeof(int), cudaMemcpyDeviceToHost));
    LLAMA_CUDA_TRY(cudaMemset(m->d_err, 0, sizeof(int)));
    if (e & LLAMA_DEVERR_TIMEOUT) return LLAMA_ERR_TIMEOUT;
    if (e) return LLAMA_ERR_INVALID_ARG;
    return LLAMA_OK;
}

void llama_free(llama_model* m) {
    if (!m) return;
    if (m->graph) cudaGraphExecDestroy(m->graph);
    if (m->cap_stream) cudaStreamDestroy(m->cap_stream);
    for (cudaEvent_t e : m->tp_ev)
        if (e) cudaEventDestroy(e);
    if (m->comm) cudaStreamDestroy(m->comm);
    delete m;
}

// ------------------------------------------------------------ single ops

int llama_op_rmsnorm(int32_t dtype, const float* d_x, const float* d_g, void* d_y, int32_t rows, int32_t d,
                     float eps, void* stream) {
    if (!d_x || !d_g || !d_y || rows < 0 || d <= 0 || d % 4 != 0 || d > 8192) return LLAMA_ERR_INVALID_ARG;
    if (dtype != LLAMA_F32 && dtype != LLAMA_BF16) return LLAMA_ERR_INVALID_ARG;
    return launch_rmsnorm(dtype, d_x, d_g, d_y, rows, d, eps, (cudaStream_t)stream);
}

int llama_op_gemm(int32_t dtype, const void* d_A, const void* d_W, float* d_C, int32_t M, int32_t N, int32_t K,
                  int32_t accumulate, void* stream) {
    if (!d_A || !d_W || !d_C || M <= 0 || N <= 0 || K <= 0) return LLAMA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (dtype == LLAMA_F32) return launch_gemm_simt(dtype, d_A, d_W, d_C, M, N, K, accumulate ? 1 : 0, st);
    if (dtype != LLAMA_BF16) return LLAMA_ERR_INVALID_ARG;
    if (K % 64 != 0 || N % 16 != 0 || (reinterpret_cast<uintptr_t>(d_C) & 15u)) return LLAMA_ERR_INVALID_ARG;
    if (accumulate && N % 32 != 0) return LLAMA_ERR_INVALID_ARG;
    TcGemm g;
    g.A = d_A;
    g.B = d_W;
    g.rowsA = M;
    g.rowsB = N;
    g.K = K;
    g.splits = 1;
    g.swap = 0;
    EpiArgs a;
    memset(&a, 0, sizeof(a));
    a.M = M;
    a.N = N;
    a.out = d_C;
    a.ld_out = N;
    int* err = nullptr;
    int rc = op_error_word(&err);
    if (rc) return rc;
    return launch_gemm_tc(g, accumulate ? EPI_RESID : EPI_F32, a, err, st);
}

int llama_op_attention_prefill(int32_t dtype, const void* d_q, const void* d_k, const void* d_v, void* d_o,
                               int32_t B, int32_t H, int32_t S, int32_t head_dim, int32_t kv_stride, void* stream) {
    if (!d_q || !d_k || !d_v || !d_o || B <= 0 || H <= 0 || S <= 0 || kv_stride < S) return LLAMA_ERR_INVALID_ARG;
    if (dtype == LLAMA_F32)
        return launch_attention_prefill_simt(dtype, d_q, d_k, d_v, d_o, B, H, H, S, head_dim, kv_stride,
                                             (cudaStream_t)stream);
    if (dtype != LLAMA_BF16) return LLAMA_ERR_INVALID_ARG;
    int* err = nullptr;
    int rc = op_error_word(&err);
    if (rc) return rc;
    int* sched = nullptr;
    if ((rc = op_attn_sched(&sched))) return rc;
    return launch_attention_prefill_tc(d_q, d_k, d_v, d_o, B, H, H, S, head_dim, kv_stride, err, sched,
                                       (cudaStream_t)stream);
}

uint64_t llama_op_attention_decode_work_bytes(int32_t B, int32_t H, int32_t max_len, int32_t head_dim) {
    if (B <= 0 || H <= 0 || max_len <= 0 || head_dim <= 0) return 0;
    return attention_decode_work_bytes(B, H, max_len, head_dim);
}

int llama_op_attention_decode(int32_t dtype, const void* d_q, const void* d_k, const void* d_v, void* d_o, int32_t B,
                              int32_t H, int32_t len, int32_t head_dim, int32_t kv_stride, void* d_work,
                              uint64_t work_bytes, void* stream) {
    if (!d_q || !d_k || !d_v || !d_o || !d_work || B <= 0 || H <= 0 || len <= 0 || kv_stride < len)
        return LLAMA_ERR_INVALID_ARG;
    if (dtype != LLAMA_F32 && dtype != LLAMA_BF16) return LLAMA_ERR_INVALID_ARG;
    if (work_bytes < attention_decode_work_bytes(B, H, len, head_dim)) return LLAMA_ERR_OOM;
    int* err = nullptr;
    int rc = op_error_word(&err);
    if (rc) return rc;
    if ((rc = attention_decode_clear((float*)d_work, B, H, len, head_dim, (cudaStream_t)stream))) return rc;
    return launch_attention_decode(dtype, d_q, d_k, d_v, d_o, B, H, H, len, nullptr, head_dim, kv_stride,
                                   (float*)d_work, attention_decode_counters((float*)d_work, B, H, len, head_dim),
                                   err, (cudaStream_t)stream);
}

int llama_debug_gemm_timeout(void* stream) {
    // 128 x 256 x 64 GEMM whose only activation tile is never requested: the
    // MMA warp's bounded wait on it must expire and the kernel must leave
    // cleanly with LLAMA_DEVERR_TIMEOUT in the error word.
    cudaStream_t st = (cudaStream_t)stream;
    int* err = nullptr;
    int rc = op_error_word(&err);
    if (rc) return rc;
    const size_t a_bytes = 128 * 64 * 2, w_bytes = 256 * 64 * 2, c_bytes = 128 * 256 * 4;
    // operands of the self-test (zeros)
    void* buf = nullptr;
    LLAMA_CUDA_TRY(cudaMallocAsync(&buf, a_bytes + w_bytes + c_bytes, st));
    LLAMA_CUDA_TRY(cudaMemsetAsync(buf, 0, a_bytes + w_bytes + c_bytes, st));
    LLAMA_CUDA_TRY(cudaMemsetAsync(err, 0, sizeof(int), st));
    TcGemm g;
    g.A = buf;
    g.B = (uint8_t*)buf + a_bytes;
    g.rowsA = 128;
    g.rowsB = 256;
    g.K = 64;
    g.splits = 1;
    g.swap = 0;
    g.test_skip_load = 1;
    EpiArgs a;
    memset(&a, 0, sizeof(a));
    a.M = 128;
    a.N = 256;
    a.out = (float*)((uint8_t*)buf + a_bytes + w_bytes);
    a.ld_out = 256;
    rc = launch_gemm_tc(g, EPI_F32, a, err, st);
    int e = 0;
    LLAMA_CUDA_TRY(cudaMemcpyAsync(&e, err, sizeof(int), cudaMemcpyDeviceToHost, st));
    LLAMA_CUDA_TRY(cudaStreamSynchronize(st));
    LLAMA_CUDA_TRY(cudaFreeAsync(buf, st));
    LLAMA_CUDA_TRY(cudaMemsetAsync(err, 0, sizeof(int), st));
    LLAMA_CUDA_TRY(cudaStreamSynchronize(st));
    if (rc) return rc;
    return (e & LLAMA_DEVERR_TIMEOUT) ? LLAMA_ERR_TIMEOUT : LLAMA_OK;
}

int llama_op_last_error(void) {
    int* err = nullptr;
    int rc = op_error_word(&err);
    if (rc) return rc;
    LLAMA_CUDA_TRY(cudaDeviceSynchronize());
    int e = 0;
    LLAMA_CUDA_TRY(cudaMemcpy(&e, err, sizeof(int), cudaMemcpyDeviceToHost));
    LLAMA_CUDA_TRY(cudaMemset(err, 0, sizeof(int)));
    LLAMA_CUDA_TRY(cudaDeviceSynchronize());
    if (e & LLAMA_DEVERR_TIMEOUT) return LLAMA_ERR_TIMEOUT;
    if (e) return LLAMA_ERR_INVALID_ARG;
    return LLAMA_OK;
}

int llama_op_argmax(const float* d_logits, int32_t rows, int32_t n, int32_t* d_out, void* stream) {
    if (!d_logits || !d_out || rows < 0 || n <= 0) return LLAMA_ERR_INVALID_ARG;
    return launch_argmax(d_logits, rows, n, n, d_out, (cudaStream_t)stream);
}

int64_t llama_kernel_launches(void) { return g_launches.load(); }

int llama_step_timeline(llama_model* m, uint64_t* h_out, int64_t n, int32_t* ctas, int32_t* phases) {
    if (!m || m->cfg.dtype != LLAMA_BF16) return LLAMA_ERR_INVALID_ARG;
    const int P = 3 + 5 * m->cfg.n_layers, G = decode_step_ctas();
    if (ctas) *ctas = G;
    if (phases) *phases = P;
    const int64_t need = (int64_t)G * P * 2;
    if (!h_out) return LLAMA_OK;
    if (n < need) return LLAMA_ERR_INVALID_ARG;
    LLAMA_CUDA_TRY(cudaMemcpy(h_out, m->step_timeline, (size_t)need * 8, cudaMemcpyDeviceToHost));
    return LLAMA_OK;
}

int llama_profile_enable(int32_t on) {
    prof::on = on != 0;
    return LLAMA_OK;
}

void llama_profile_reset(void) {
    prof::flush();
    prof::entries.clear();
}

int llama_profile_count(void) {
    prof::flush();
    return (int)prof::entries.size();
}

int llama_profile_entry(int32_t i, const char** name, double* ms, int64_t* launches, int64_t* calls,
                        double* bytes, double* flops) {
    if (i < 0 || i >= (int)prof::entries.size()) return LLAMA_ERR_INVALID_ARG;
    const prof::Entry& e = prof::entries[i];
    if (name) *name = e.name.c_str();
    if (ms) *ms = e.ms;
    if (launches) *launches = e.launches;
    if (calls) *calls = e.calls;
    if (bytes) *bytes = e.bytes;
    if (flops) *flops = e.flops;
    return LLAMA_OK;
}

}  // extern "C"
