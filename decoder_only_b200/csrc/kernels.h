// Internal launchers of the llama_b200 kernels (host side).  Every function
// queues work on `st` and returns a llama_status.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "llama_b200.h"

struct EpiArgs;

// init.cu
int launch_init_matrix(int dtype, void* dst, int K, int N_log, int blk, int blk_stride, int row_off,
                       int rowmajor_nk, uint32_t seed, uint32_t tensor_id, double scale, cudaStream_t st);
// block n in [n0, n0 + N_loc), k in [k0, k0 + K_loc) of a (K_full, N_full) logical matrix
int launch_init_shard(int dtype, void* dst, int K_full, int N_full, int k0, int K_loc, int n0, int N_loc, int blk,
                      int blk_stride, int row_off, int rowmajor_nk, uint32_t seed, uint32_t tensor_id, double scale,
                      cudaStream_t st);
int launch_fill_f32(float* dst, float v, int64_t n, cudaStream_t st);
// c = b + W beta per row of W [rows, K] (the bias variant's folded bias)
int launch_bias_fold(int dtype, const void* W, int rows, int K, const float* beta, const float* b, float* c,
                     cudaStream_t st);

// norm.cu
// y = x / rms(x) * g (+ beta, the bias variant's shift, when beta is not NULL)
int launch_rmsnorm(int dtype, const float* x, const float* g, void* y, int rows, int d, float eps,
                   cudaStream_t st, const float* beta = nullptr);
int launch_embed(int dtype, const int32_t* tok, const void* E, float* x, int rows, int d, int vocab, int* err,
                 cudaStream_t st);
int launch_argmax(const float* logits, int rows, int n, int64_t ld, int32_t* out, cudaStream_t st);
int argmax_split_chunks(int n);
// part: int2 [rows][argmax_split_chunks(n)]; counters: int [rows], zero between launches
int launch_argmax_split(const float* logits, int rows, int n, int64_t ld, int32_t* out, int2* part, int* counters,
                        cudaStream_t st);

// simt.cu  (fp32 storage path and shared epilogue passes)
int launch_gemm_simt(int dtype, const void* A, const void* W, float* C, int M, int N, int K, int accumulate,
                     cudaStream_t st);
int launch_epilogue_from_f32(int dtype, int mode, const float* C, int ldc, const EpiArgs& a, cudaStream_t st);
int launch_attention_prefill_simt(int dtype, const void* q, const void* k, const void* v, void* o, int B,
                                  int H, int Hkv, int S, int hd, int kv_stride, cudaStream_t st);
int attention_prepare();  // sets kernel attributes; call before any stream capture

// attn_tc.cu  (bf16 tcgen05 causal flash attention, head_dim 64 or 128)
// pages (device, [B][pps] page ids) != NULL: k and v are page pools of n_pages pages [Hkv][128][hd]
// sched: two device ints, zero before the first launch and left zero by each
// launch (the work-item counter); launches sharing them must not overlap
int launch_attention_prefill_tc(const void* q, const void* k, const void* v, void* o, int B, int H, int Hkv, int S,
                                int hd, int kv_stride, int* err, int* sched, cudaStream_t st,
                                const int* pages = nullptr, int pps = 0, int n_pages = 0);
int attention_tc_prepare();

// decode.cu
uint64_t attention_decode_work_bytes(int B, int H, int max_len, int hd);
// counters: int [B*H], zero before the launch (each launch leaves them zero)
int launch_attention_decode(int dtype, const void* q, const void* k, const void* v, void* o, int B, int H,
                            int Hkv, int len, const int* d_len_minus1, int hd, int kv_stride, float* work,
                            int* counters, int* err, cudaStream_t st);
int* attention_decode_counters(float* work, int B, int H, int max_len, int hd);
int attention_decode_clear(float* work, int B, int H, int len, int hd, cudaStream_t st);
int attention_decode_prepare();
int op_error_word(int** p);   // error word of the standalone ops

// gemm_tc.cu  (bf16 tcgen05 GEMM)
struct TcGemm {
    // C-tile roles: rows of the 128-row operand "A" map to TMEM lanes.
    const void* A;  // bf16 [rowsA, K]
    const void* B;  // bf16 [rowsB, K]
    int rowsA, rowsB, K;
    int splits;     // split-K factor (decode only)
    int swap;       // must be 0 (decode projections run in decode_step.cu)
    int test_skip_load = 0;   // test hook (llama_debug_gemm_timeout)
};
int launch_gemm_tc(const TcGemm& g, int mode, const EpiArgs& a, int* err, cudaStream_t st);
int gemm_tc_pick_splits(int rowsA, int K);

// decode_step.cu  (one cooperative kernel per greedy decode step, bf16)
// At most this many CTAs run the fused decode step (one per SM), each with
// this many warps working on attention.
constexpr int STEP_MAX_CTAS = 160;
constexpr int STEP_ATTN_WARPS = 6;
// Partial-sum slots per output feature of a projection with `mblk` 128-row
// blocks when its (block, k-block) iterations are cut into `ctas` equal
// contiguous ranges: no block is touched by more ranges than this.
__host__ __device__ inline int step_slots(int mblk, int ctas) { return (ctas + mblk - 1) / mblk + 1; }

struct StepArgs {
    const CUtensorMap* maps;      // device table: 4 per layer (W_qkv, W_o, W_gu, W_d), head, xg, attn, act, xg2
    const float* const* gains;    // device table [2L + 1]: g_attn[l], g_ffn[l], ..., g_final
    const float* const* biases;   // bias variant: device table [4L] (b_qkv + W_qkv beta_attn, b_o,
                                  // b_gu + W_gu beta_ffn, b_d per layer), or NULL
    const __nv_bfloat16* embed;
    __nv_bfloat16* kv;            // layer l: K at kv + 2l * kv_layer, V at kv + (2l + 1) * kv_layer
    size_t kv_layer;
    float* trunk;
    __nv_bfloat16* xg;            // g (.) x of the attention / final norm, bf16 [B][d]
    __nv_bfloat16* xg2;           // g (.) x of the FFN norm, bf16 [B][d]
    float* ssq;                   // [2][64][32] per 128-feature block sums of squares (attention, FFN norm)
    __nv_bfloat16 *q, *attn, *act;
    float* logits;
    float* partial;               // split-K partials, one region per projection kind
    long long part_off[5];        // qkv, o, gate/up, down, head (floats)
    int* counters;                // arrival counters, one region per projection kind
    int cnt_off[5];
    float* attn_work;             // attention partials [B*H][ranges per pair][hd + 2]
    int* attn_cnt;                // [B*H]
    int2* amax_part;              // [B][ceil(V/2048)]
    int* amax_cnt;                // [B + 1]
    int32_t* tok;
    int* d_pos;
    int* err;
    unsigned int* bar;            // step synchronisation words [decode_step_sync_words(L)]
    unsigned long long* timeline; // optional: per CTA and phase, start / end %globaltimer stamps
    const float2* rope;
    int L, d, h, V, H, hd, B, smax;
    int Hkv;                      // key/value heads (query head h uses h / (H / Hkv))
    float eps;
    const int* pages;             // paged KV cache: page table [B][pps] (device), or NULL (contiguous)
    int pps;
};
int decode_step_prepare();
int launch_decode_step(const StepArgs& a, cudaStream_t st);
int decode_step_maps(CUtensorMap* host_maps, const void* const* w, int L, const void* head, const void* xg,
                     const void* attn, const void* act, const void* xg2, int B, int qkv_rows, int d, int h, int V);
// Grid of the fused decode step, and the partial / counter regions for batch B
int decode_step_ctas();
inline size_t decode_step_sync_words(int L) { return 128 + 256 * (size_t)(L + 1); }
long long decode_step_layout(int ctas, int qkv_rows, int d, int h, int V, int B, long long part_off[5],
                             int cnt_off[5]);
// 2-D K-major bf16 tensor map, box (64, box_rows), 128-byte swizzle, zero fill
int tc_make_map_2d(CUtensorMap* map, const void* ptr, int rows, int K, int box_rows);
int tc_num_sms();
int gemm_tc_prepare();  // sets kernel attributes; call before any stream capture
