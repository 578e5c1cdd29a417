// params.h -- launch parameters shared by the host API and the kernels.
#pragma once
#include <cstdint>
#include <cuda.h>

namespace pf {

struct FwdParams {
    const uint16_t *k;            // [T][G][D] this call's keys (for the cache write)
    const uint16_t *v;            // [T][G][D]
    uint16_t *out;                // [T][H][D]
    uint16_t *cache;              // [NB][2][bs][G][D], or nullptr: no cache write (plain prefill only)
    const int32_t *cu_seqlens;    // [B+1]
    const int32_t *context_lens;  // [B] or nullptr (plain prefill)
    const int32_t *block_table;   // [B][mbps]
    int32_t *status;              // nullable
    int num_seqs;
    int n_head;
    int n_kv_head;
    int group;                    // n_head / n_kv_head
    int total;                    // rows of q/k/v/out
    int num_blocks;
    int mbps;                     // max_blocks_per_seq
    int block_size;
    int max_q;                    // bound on every sequence (chunk) length
    float scale_log2;             // scale * log2(e)
    int test_stall;               // test hook: withhold one Q tile (see prefill_test_inject_stall)
    int max_ctx;                  // bound on every context length (chunked prefill; 0 otherwise)
    int window;                   // sliding window: row P sees keys P-window+1 .. P (<= 0: none)
    // split-KV: kv ranges split into up to nsplit parts; the partial results go to
    // part_o [nsplit][n_head][D / 4][total] float4 (fp32, unnormalised; the rows of
    // one 4-column chunk contiguous, so that a warp's 32 rows store 512
    // contiguous bytes) and part_ml [nsplit][n_head][total][2] (running max in
    // log2 units, exp-sum), and
    // part_nsp [total] holds, for every row of a valid sequence, its pair's split
    // count tagged with this launch's epoch ((epoch << 4) | splits), so that the
    // merge kernel skips rows that this launch did not split (or did not reach)
    int nsplit = 1;
    float *part_o = nullptr;
    float *part_ml = nullptr;
    uint32_t *part_nsp = nullptr;
    uint32_t epoch = 0;
    // per-kv-head factors folded into the scores (k_fold[g]) and into the output
    // (v_fold[g]), or nullptr (factor 1): a chunked prefill over an FP8 cache
    // stages e4m3 code values (exact in bf16) and applies the cache's scales here
    const float *k_fold = nullptr;
    const float *v_fold = nullptr;
    // chunked prefill over an FP8 cache (the call has stored the chunk's codes
    // already): the kernel reads every key and value as e4m3 codes -- the prefix
    // through the block table from the FP8 pool (tensor map `cache`), the chunk's
    // own rows from a dense copy of their codes (tensor maps `k`, `v`) -- and runs
    // its products on f16 operands; cache (bf16) is nullptr
    int fp8 = 0;
};

struct TensorMaps {
    CUtensorMap q;      // {64, H, T, D/64} (chunk outermost), box {64, 1, 128, D/64}
    CUtensorMap k;      // {64, G, T, D/64}, box {64, 1, 128, D/64}; FP8: uint8 {D, G, T, 1}, box {D, 1, 128, 1}
    CUtensorMap v;      // as k
    CUtensorMap cache;  // {D, G, bs, 2*NB}, box {64, 1, bs, 1}; FP8: uint8, box {D, 1, bs, 1}
};

// Launchers (defined per kernel file); return a cudaError_t value.
// Pipelined warp-specialised kernel (prefill_fwd.cu) and the sizes it takes.
int launch_fwd(const TensorMaps &maps, const FwdParams &p, int head_dim, void *stream);
bool fwd_pipelined_supported(const FwdParams &p, int head_dim);
// Split count for the pipelined kernel (1 = no split) and its workspace bytes.
int fwd_choose_splits(const FwdParams &p);
size_t fwd_split_workspace_bytes(const FwdParams &p, int head_dim);
// exp2_fma2 (the FMA-pipe exponential of the pipelined kernel) applied to n floats (test hook).
int launch_exp2_fma2_probe(const float *x, float *y, int n, void *stream);
// One-CTA-per-query-block kernel (prefill_fwd_v0.cu): no size limits.
int launch_fwd_v0(const TensorMaps &maps, const FwdParams &p, int head_dim, void *stream);

// Host path shared by the C entry points (api.cu).  scratch / scratch_bytes:
// caller-supplied split-KV scratch (nullptr: the library's own workspace); the
// split count is lowered until the partials fit scratch_bytes (1 needs none).
// window: sliding window of that many keys (0: plain causal).  cache8 (with
// k_scale / v_scale): the K/V rows go to this FP8 cache instead of `cache`
// (plain prefill only; cache is then nullptr): the attention kernel runs
// without its cache writer and the FP8 store kernel follows on the stream.
// k_fold / v_fold: per-kv-head factors applied to the scores and to the output
// (FwdParams::k_fold / v_fold); the call then needs the pipelined kernel.
int run_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v, int total, const int32_t *cu,
                const int32_t *ctx_lens, bool chunked, int num_seqs, int max_q, long long max_ctx, int n_head,
                int n_kv_head, int head_dim, float scale, uint16_t *out, uint16_t *cache, int num_blocks,
                const int32_t *bt, int mbps, int bs, int32_t *status, struct CUstream_st *stream, void *scratch,
                size_t scratch_bytes, int window = 0, uint8_t *cache8 = nullptr, const float *k_scale = nullptr,
                const float *v_scale = nullptr, const float *k_fold = nullptr, const float *v_fold = nullptr);

// SM count of the current device (cached per device ordinal).
int device_sm_count();

}  // namespace pf
