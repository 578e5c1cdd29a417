// decode.h -- launch parameters of the paged decode kernels (decode.cu).
#pragma once
#include <cuda.h>

#include <cstdint>

namespace pf {

// At most this many key splits (work units) per sequence; longer contexts get
// longer units (decode_keys_per_unit).
constexpr int kDecodeMaxUnits = 64;
// Sequences per decode call (their context lengths and unit counts are kept in
// shared memory by every CTA).
constexpr int kDecodeMaxSeqs = 2048;

struct DecodeParams {
    const uint16_t *q;            // [B][n_head][D]   the new token's queries
    const uint16_t *k;            // [B][n_kv_head][D] its keys
    const uint16_t *v;            // [B][n_kv_head][D] its values
    uint16_t *out;                // [B][n_head][D]
    uint16_t *cache;              // [NB][2][bs][n_kv_head][D]
    const int32_t *context_lens;  // [B] cached tokens before the new one
    const int32_t *block_table;   // [B][mbps]
    int32_t *status;              // nullable
    int num_seqs, n_head, n_kv_head;
    int num_blocks, mbps, block_size;
    int max_ctx;                  // bound on every context length (sizes the grid)
    int keys_per_unit;            // keys per work unit (a multiple of the 64-key tile)
    int max_units;                // cdiv(max_ctx + 1, keys_per_unit)
    float scale_log2;             // scale * log2(e)
    // FP8 (e4m3) cache: codes [NB][2][bs][n_kv_head][D] in cache8 (cache unused);
    // the value of a code is code_value * k_scale[g] (K) or * v_scale[g] (V)
    uint8_t *cache8;
    const float *k_scale, *v_scale;
    // units' partials when a sequence has more than one unit:
    // part_o [max_units][B][n_head][D] (fp32, unnormalised), part_ml [..][2] (max in log2 units, sum)
    float *part_o;
    float *part_ml;
    // whole-page kernel: its grid (CTAs; the call's 16-key steps are divided
    // evenly over them), and [num_seqs + 1] steps before each sequence (written
    // by the kernel for the merge kernel).  Its partial rows are
    // [piece id][n_head / slabs] (see get_piece), at most
    // grid * n_head / slabs + num_seqs * n_head rows.
    int grid = 0;
    int32_t *seg_cum = nullptr;
};

int decode_keys_per_unit(int max_ctx);
int launch_decode(const DecodeParams &p, int head_dim, bool fp8, void *stream);
// The whole-page kernel (n_kv_head a multiple of 8; head_dim 128 for the FP8
// cache): tm maps the cache as [2 * num_blocks][n_kv_head][block_size][head_dim]
// (innermost last; the token dimension is strided past the kv heads), boxes of
// 16 tokens x 8 kv heads x 128 bytes with 128-byte swizzle.
int launch_decode_tma(const DecodeParams &p, const CUtensorMap *tm, int head_dim, bool fp8, void *stream);

// FP8 store of a call's K/V rows into their cache slots (decode.cu).
// Every member has a default, so that a call site that does not know a
// member (e.g. the optional dense copy) leaves it null, never uninitialised.
struct Fp8StoreParams {
    const uint16_t *k = nullptr, *v = nullptr;  // [T][n_kv_head][D]
    const int32_t *cu_seqlens = nullptr;        // [B + 1]
    const int32_t *context_lens = nullptr;      // [B] or nullptr
    const float *k_scale = nullptr, *v_scale = nullptr;
    uint8_t *cache8 = nullptr;                  // [NB][2][bs][n_kv_head][D]
    uint8_t *dense_k8 = nullptr, *dense_v8 = nullptr;  // nullable: the same codes packed like k / v
    const int32_t *block_table = nullptr;       // [B][mbps]
    int32_t *status = nullptr;
    int total = 0, num_seqs = 0, n_kv_head = 0, num_blocks = 0, mbps = 0, block_size = 0;
};
int launch_kv_store_fp8(const Fp8StoreParams &p, int head_dim, void *stream);


}  // namespace pf
