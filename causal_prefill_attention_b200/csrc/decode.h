// decode.h -- launch parameters of the paged decode kernels (decode.cu).
#pragma once
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
};

int decode_keys_per_unit(int max_ctx);
int launch_decode(const DecodeParams &p, int head_dim, bool fp8, void *stream);

// FP8 store of a call's K/V rows into their cache slots (decode.cu).
struct Fp8StoreParams {
    const uint16_t *k, *v;        // [T][n_kv_head][D]
    const int32_t *cu_seqlens;    // [B + 1]
    const int32_t *context_lens;  // [B] or nullptr
    const float *k_scale, *v_scale;
    uint8_t *cache8;              // [NB][2][bs][n_kv_head][D]
    const int32_t *block_table;   // [B][mbps]
    int32_t *status;
    int total, num_seqs, n_kv_head, num_blocks, mbps, block_size;
};
int launch_kv_store_fp8(const Fp8StoreParams &p, int head_dim, void *stream);

// Staging of a chunked prefill over an FP8 cache (decode.cu): sequence i's
// positions 0 .. ctx_i + n_i - 1 are read from the FP8 cache through the block
// table and widened to their e4m3 code values in bf16 (exact; no scale); the
// prefix (p < ctx_i) goes to a bf16 shadow pool whose block table gives
// sequence i the pages i * mbps2 .. i * mbps2 + mbps2 - 1, the chunk's own rows
// to k2 / v2 (packed like the call's k / v).  The bf16 chunked kernel then runs
// on them with the per-kv-head scales folded into its scores and output.
struct Fp8StageParams {
    const uint8_t *cache8;        // [NB][2][bs][G][D] codes (the chunk's rows already stored)
    const int32_t *block_table;   // [B][mbps]
    const int32_t *cu_seqlens;    // [B + 1] chunk rows
    const int32_t *context_lens;  // [B]
    uint16_t *shadow;             // [B * mbps2][2][bs][G][D] bf16
    int32_t *shadow_table;        // [B][mbps2]
    uint16_t *k2, *v2;            // [T][G][D] bf16
    int32_t *status;
    int total;                    // rows of k2 / v2 (= the call's chunk rows)
    int num_seqs, n_kv_head, num_blocks, mbps, block_size, mbps2, max_span;
};
int launch_fp8_stage(const Fp8StageParams &p, int head_dim, void *stream);

}  // namespace pf
