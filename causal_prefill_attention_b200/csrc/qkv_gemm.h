// qkv_gemm.h -- launch parameters of the projection GEMM (qkv_gemm.cu): the
// fused QKV projection, and with hq = N, hkv = 0 a plain y = x w^T into q
// (the attention's output projection W_o).
#pragma once
#include <cstdint>
#include <cstddef>
#include <cuda.h>

namespace pf {

struct QkvParams {
    uint16_t *q;        // [M][hq]  = [T][n_head][head_dim]
    uint16_t *k;        // [M][hkv] = [T][n_kv_head][head_dim]
    uint16_t *v;        // [M][hkv]
    int M, N, K;        // tokens, output features, input features
    int hq, hkv;        // n_head * head_dim, n_kv_head * head_dim
    int32_t *status;    // nullable
};

// Output tile width (256, or 192 when N allows it and the tiles fill the
// waves of a persistent grid of `sms` CTAs better); the W tensor map's box
// is tile_n rows of 64 columns.
int qkv_gemm_tile_n(int M, int N, int sms);
size_t qkv_gemm_smem_bytes(int tile_n);
int launch_qkv_gemm(const CUtensorMap &tm_x, const CUtensorMap &tm_w, const QkvParams &p, int tile_n, void *stream);

}  // namespace pf
