// prefill_fwd_v0.cu -- straightforward tcgen05 attention forward, one CTA per
// (query block of 128 rows, query head, sequence), no intra-CTA overlap.
//
// It is the correctness baseline for the pipelined kernel: every step of the
// tiled method (hncyxsy.com/news/270449 §3.2 and §4.3) runs in order:
//   TMA Q block -> for each kv block: TMA K,V -> S = Q K^T (tcgen05, fp32 in
//   TMEM) -> online softmax in registers (running row max and exp-sum, old O
//   rescaled) -> P as bf16 into TMEM -> O += P V (tcgen05, A from TMEM)
//   -> O / l to bf16 -> the block's K/V rows copied into their cache pages.
#include <cuda_runtime.h>
#include <cstdint>
#include <math_constants.h>

#include "block_rule.h"
#include "params.h"
#include "sm100.cuh"
#include "../../include/prefill.h"

namespace pf {
namespace {

constexpr int BM = 128;                  // query rows per block
constexpr int BN = 128;                  // keys per kv block
constexpr uint32_t CHUNK_BYTES = 128 * 128;  // 128 rows x 64 bf16 (one 128B-swizzled chunk)

template <int D>
struct V0Layout {
    static constexpr int NCH = D / 64;
    static constexpr uint32_t TILE = NCH * CHUNK_BYTES;   // one 128 x D bf16 tile
    static constexpr uint32_t Q = 0, K = TILE, V = 2 * TILE;
    static constexpr uint32_t BAR_LOAD = 3 * TILE, BAR_MMA = BAR_LOAD + 8, TMEM_SLOT = BAR_LOAD + 16;
    static constexpr uint32_t BYTES = BAR_LOAD + 64;
};

template <int D>
__global__ void __launch_bounds__(128, 1)
prefill_fwd_v0_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_cache,
                      const FwdParams p) {
    using L = V0Layout<D>;
    constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false, false);
    constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, false, true);

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);

    const int qb = blockIdx.x, h = blockIdx.y, i = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5;

    const int c0 = p.cu_seqlens[i];
    const int n = p.cu_seqlens[i + 1] - c0;
    const int ctx = p.context_lens ? p.context_lens[i] : 0;
    const bool bad_len = n < 0 || n > p.max_q || c0 < 0 || c0 + n > p.total;
    const bool bad_ctx = ctx < 0 || (long long)ctx + n > (long long)p.mbps * p.block_size;
    if (bad_len || bad_ctx) {
        if (qb == 0 && h == 0 && tid == 0) report(p.status, bad_len ? PREFILL_ERR_SHAPE : PREFILL_ERR_BLOCK_TABLE);
        return;
    }
    if (qb * BM >= n) return;
    const int g = h / p.group;
    const int bs = p.block_size;

    const uint32_t sQ = base + L::Q, sK = base + L::K, sV = base + L::V;
    const uint32_t bar_load = base + L::BAR_LOAD, bar_mma = base + L::BAR_MMA;

    if (tid == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_cache);
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(base + L::TMEM_SLOT, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(gbase + L::TMEM_SLOT);
    const uint32_t tS = tmem;          // S (fp32, 128 cols); P (bf16x2, 64 cols) aliases its start
    const uint32_t tO = tmem + 128;    // O (fp32, D cols)
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    uint32_t ph_load = 0, ph_mma = 0;
    int ok = 1;

    // ---- Q block
    if (tid == 0) {
        mbar_expect_tx(bar_load, L::TILE);
        tma_load_4d(sQ, &tm_q, bar_load, 0, h, c0 + qb * BM, 0);
    }
    ok = __syncthreads_and(mbar_wait(bar_load, ph_load));
    ph_load ^= 1;

    const int nkv = num_kv_blocks(qb, ctx, n, BM, BN);
    const int j0 = first_kv_block(qb, ctx, n, BM, BN, p.window);  // 0 without a sliding window
    const int row = tid;  // query row of this thread inside the block (TMEM lane)
    float m_run = -CUDART_INF_F, l_run = 0.f;

    for (int j = j0; j < nkv && ok; ++j) {
        const KvBlock kb = kv_block(qb, j, ctx, n, BM, BN, p.window);
        // ---- K, V block (prefix: gathered page by page from the cache)
        if (tid == 0) {
            if (kb.prefix) {
                const int pages = cdiv(kb.lim_const, bs);
                mbar_expect_tx(bar_load, 2u * L::NCH * pages * bs * 128u);
                for (int pg = 0; pg < pages; ++pg) {
                    const int lp = kb.key_begin / bs + pg;
                    int page = p.block_table[(size_t)i * p.mbps + lp];
                    if (page < 0 || page >= p.num_blocks) {
                        report(p.status, PREFILL_ERR_BLOCK_TABLE);
                        page = p.num_blocks;  // outside the tensor map: TMA fills zeros
                    }
#pragma unroll
                    for (int ch = 0; ch < L::NCH; ++ch) {
                        const uint32_t off = ch * CHUNK_BYTES + pg * bs * 128;
                        tma_load_4d(sK + off, &tm_cache, bar_load, ch * 64, g, 0, page * 2 + 0);
                        tma_load_4d(sV + off, &tm_cache, bar_load, ch * 64, g, 0, page * 2 + 1);
                    }
                }
            } else {
                mbar_expect_tx(bar_load, 2u * L::TILE);
                tma_load_4d(sK, &tm_k, bar_load, 0, g, c0 + kb.src_row, 0);
                tma_load_4d(sV, &tm_v, bar_load, 0, g, c0 + kb.src_row, 0);
            }
        }
        ok = __syncthreads_and(mbar_wait(bar_load, ph_load));
        ph_load ^= 1;
        if (!ok) break;
        if (kb.prefix && !kb.full) {
            // rows past the end of the prefix hold stale or unwritten data: zero
            // them so that a masked (P = 0) row can never contribute NaN * 0.
            const int first = kb.lim_const;
            const int units = (BN - first) * 8 * L::NCH * 2;
            for (int u = tid; u < units; u += 128) {
                const int t = u / ((BN - first) * 8 * L::NCH);
                const int rem = u % ((BN - first) * 8 * L::NCH);
                const int ch = rem / ((BN - first) * 8);
                const int rr = first + (rem % ((BN - first) * 8)) / 8;
                const int un = rem % 8;
                uint8_t *dst = gbase + (t ? L::V : L::K) + ch * CHUNK_BYTES + rr * 128 + un * 16;
                *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncthreads();
        }

        // ---- S = Q K^T
        tc_fence_after();
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * CHUNK_BYTES + (kk & 3) * 32;
                mma_ss(tS, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(sK + off, 16, 1024),
                       IDESC_QK, kk > 0);
            }
            tc_commit(bar_mma);
        }
        ok = __syncthreads_and(mbar_wait(bar_mma, ph_mma));
        ph_mma ^= 1;
        if (!ok) break;
        tc_fence_after();

        // ---- online softmax on this thread's row
        float x[BN];
        {
            uint32_t r[32];
#pragma unroll
            for (int c4 = 0; c4 < BN / 32; ++c4) {
                tmem_ld32(tS + lane_off + c4 * 32, r);
#pragma unroll
                for (int c = 0; c < 32; ++c) x[c4 * 32 + c] = __uint_as_float(r[c]);
            }
        }
        const int lim = kb.full ? BN : col_limit(kb, row, BN);
        const int lo = kb.full ? 0 : col_lo(kb, row, BN);
        float mt = -CUDART_INF_F;
#pragma unroll
        for (int c = 0; c < BN; ++c) {
            x[c] = (c >= lo && c < lim) ? x[c] * p.scale_log2 : -CUDART_INF_F;
            mt = fmaxf(mt, x[c]);
        }
        // a row with nothing visible yet (possible under a sliding window) keeps
        // a finite floor, so that the first visible key rescales by exactly 0
        const float m_new = fmaxf(fmaxf(m_run, mt), -1e30f);
        const float alpha = ex2(m_run - m_new);
        float sum = 0.f;
        {
            uint32_t pw[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float p0 = ex2(x[half * 64 + 2 * c] - m_new);
                    const float p1 = ex2(x[half * 64 + 2 * c + 1] - m_new);
                    sum += p0 + p1;
                    pw[c] = pack_bf16x2(p0, p1);
                }
                tmem_st32(tS + lane_off + half * 32, pw);
            }
        }
        l_run = l_run * alpha + sum;
        m_run = m_new;
        if (j > j0) {
            uint32_t r[32];
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                tmem_ld32(tO + lane_off + cc * 32, r);
#pragma unroll
                for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
                tmem_st32(tO + lane_off + cc * 32, r);
            }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- O += P V
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
                mma_ts(tO, tS + kk * 8, smem_desc_sw128(sV + kk * 2048, CHUNK_BYTES, 1024), IDESC_PV,
                       (j > j0 || kk > 0) ? 1u : 0u);
            tc_commit(bar_mma);
        }
        ok = __syncthreads_and(mbar_wait(bar_mma, ph_mma));
        ph_mma ^= 1;
    }
    if (!ok && tid == 0) report(p.status, PREFILL_ERR_TIMEOUT);

    // ---- epilogue: O / l -> bf16 rows of out
    tc_fence_after();
    const int a = qb * BM + row;
    if (ok) {
        const float inv_l = 1.f / l_run;
        uint16_t *dst = p.out + ((size_t)(c0 + a) * p.n_head + h) * D;
        uint32_t r[32];
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
            tmem_ld32(tO + lane_off + cc * 32, r);
            uint32_t w[16];
#pragma unroll
            for (int c = 0; c < 16; ++c)
                w[c] = pack_bf16x2(__uint_as_float(r[2 * c]) * inv_l, __uint_as_float(r[2 * c + 1]) * inv_l);
            if (a < n) {
                uint4 *d4 = reinterpret_cast<uint4 *>(dst + cc * 32);
#pragma unroll
                for (int c = 0; c < 4; ++c) d4[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
            }
        }
    }

    // ---- paged KV write for this block's tokens (one query head per kv group does it)
    if (ok && (h % p.group) == 0 && a < n) {
        const int P = ctx + a;
        const int page = p.block_table[(size_t)i * p.mbps + P / bs];
        if (page < 0 || page >= p.num_blocks) {
            report(p.status, PREFILL_ERR_BLOCK_TABLE);
        } else {
            const size_t G = p.n_kv_head;
            const size_t slot = P % bs;
            const uint4 *ks = reinterpret_cast<const uint4 *>(p.k + ((size_t)(c0 + a) * G + g) * D);
            const uint4 *vs = reinterpret_cast<const uint4 *>(p.v + ((size_t)(c0 + a) * G + g) * D);
            uint4 *kd = reinterpret_cast<uint4 *>(p.cache + ((((size_t)page * 2 + 0) * bs + slot) * G + g) * D);
            uint4 *vd = reinterpret_cast<uint4 *>(p.cache + ((((size_t)page * 2 + 1) * bs + slot) * G + g) * D);
#pragma unroll
            for (int c = 0; c < D * 2 / 16; ++c) {
                kd[c] = ks[c];
                vd[c] = vs[c];
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

template <int D>
int launch(const TensorMaps &maps, const FwdParams &p, void *stream) {
    using L = V0Layout<D>;
    const size_t smem = L::BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(prefill_fwd_v0_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return (int)e;
    dim3 grid(cdiv(p.max_q, BM), p.n_head, p.num_seqs);
    prefill_fwd_v0_kernel<D><<<grid, 128, smem, (cudaStream_t)stream>>>(maps.q, maps.k, maps.v, maps.cache, p);
    return (int)cudaGetLastError();
}

}  // namespace

int launch_fwd_v0(const TensorMaps &maps, const FwdParams &p, int head_dim, void *stream) {
    if (head_dim == 64) return launch<64>(maps, p, stream);
    return launch<128>(maps, p, stream);
}

}  // namespace pf
