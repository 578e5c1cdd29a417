// qkv_gemm.cu -- the fused QKV projection that feeds the attention.
//
// hncyxsy.com/news/270449 §4.1: the W_q, W_k and W_v blocks are concatenated
// so that one large GEMM reads the activations x once, and its (s, (H + 2G) d)
// output is cut by columns into Q, K and V; §2.2: each is reshaped to
// (s, heads, head_dim), head_dim last.  Here y = x W^T with W stored one row
// per output feature ([N][hidden], the Q block's rows first), and the
// epilogue writes the Q, K and V column ranges straight into the [T][H][d] /
// [T][G][d] tensors the attention call reads.  The same kernel runs the
// output projection W_o after the attention (§3.3: the heads' outputs merged
// by flattening (s, n_head, head_dim), then one plain GEMM): there every
// column goes to one output, q = y [T][hidden].
//
// Design (a dense contraction: tcgen05 tensor cores):
//  * persistent grid, one CTA per SM; 128 x BN output tiles (BN 256, or 192
//    when the output width allows it and the tiles then fill the last wave of
//    CTAs better), K in steps of 64, taken in grouped order (tile_coords) so
//    that operands are re-read from L2;
//  * warp 0 loads A (x, 128 x 64) and B (W, BN x 64) tiles by TMA, 128-byte
//    swizzled, into a 4-stage (BN 256) or 5-stage (BN 192) ring; warp 1 issues
//    tcgen05.mma (M 128, N BN, K 16) with the fp32 accumulator in TMEM, two
//    accumulators so that the epilogue of one tile overlaps the MMAs of the next;
//  * warps 2-5 drain the accumulator (tcgen05.ld, 32 rows each), round to bf16
//    and store each 32-column slice into q, k or v;
//  * every mbarrier wait is bounded (about a second) and raises a CTA abort
//    flag; the producer drains its copies before exit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/prefill.h"
#include "block_rule.h"
#include "qkv_gemm.h"
#include "sm100.cuh"

namespace pf {
namespace {

constexpr int GBM = 128, GBK = 64;
constexpr int GTHREADS = 192;  // warp 0: TMA, warp 1: MMA, warps 2-5: epilogue
template <int GBN>
struct GLay {
    static constexpr int GST = GBN == 256 ? 4 : 5;           // ring stages
    static constexpr uint32_t A_TILE = GBM * GBK * 2;         // 16 KB
    static constexpr uint32_t B_TILE = GBN * GBK * 2;         // 32 or 24 KB
    static constexpr uint32_t GSTAGE = A_TILE + B_TILE;
    static constexpr uint32_t G_BAR = GST * GSTAGE;
    // barriers: full[GST], empty[GST], acc_full[2], acc_empty[2]
    static constexpr int G_FULL = 0, G_EMPTY = GST, G_AFULL = 2 * GST, G_AEMPTY = 2 * GST + 2, G_NBAR = 2 * GST + 4;
    static constexpr uint32_t G_TMEM_SLOT = G_BAR + G_NBAR * 8, G_ABORT = G_TMEM_SLOT + 4;
    static constexpr uint32_t G_SMEM = G_ABORT + 4 + 1024;  // + slack to align the ring to 1024 bytes
    static_assert(G_SMEM <= 227 * 1024, "shared memory");
    static_assert(2 * GBN <= 512, "two accumulators in TMEM");
};

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *m, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

// Tile order: groups of kGroupM row tiles (128 rows of x each), and inside a
// group column tile after column tile, the group's row tiles first.  The CTAs
// working at one time then share a few x row panels and a band of W, so each
// operand tile is fetched from DRAM about once and re-read from L2 by the
// neighbouring tiles (row-major order made every wave re-read all of W).
// Measured on x [8192, 4096] x W [6144, 4096]: row-major order 1354 TFLOP/s,
// groups of 4 / 8 / 16 rows 1439 / 1398 / 1422, column-major 1312.
#ifndef PF_QKV_GROUP_M
#define PF_QKV_GROUP_M 4
#endif
constexpr int kGroupM = PF_QKV_GROUP_M;
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int &tm, int &tn) {
    const int per_group = kGroupM * tiles_n;
    const int g = t / per_group;
    const int first = g * kGroupM;
    const int rows = tiles_m - first < kGroupM ? tiles_m - first : kGroupM;
    const int r = t - g * per_group;
    tm = first + r % rows;
    tn = r / rows;
}

__device__ __forceinline__ bool gwait(uint32_t bar, uint32_t parity, volatile int *abort) {
    if (mbar_wait(bar, parity, abort)) return true;
    *abort = 1;
    return false;
}

template <int GBN>
__global__ void __launch_bounds__(GTHREADS, 1)
qkv_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                const QkvParams p) {
    using GL = GLay<GBN>;
    constexpr int GST = GL::GST;
    constexpr uint32_t A_TILE = GL::A_TILE, GSTAGE = GL::GSTAGE, G_BAR = GL::G_BAR;
    constexpr int G_FULL = GL::G_FULL, G_EMPTY = GL::G_EMPTY, G_AFULL = GL::G_AFULL, G_AEMPTY = GL::G_AEMPTY;
    constexpr uint32_t G_TMEM_SLOT = GL::G_TMEM_SLOT, G_ABORT = GL::G_ABORT;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int *abort = reinterpret_cast<volatile int *>(gbase + G_ABORT);
    auto bar = [&](int i) -> uint32_t { return base + G_BAR + 8u * i; };

    if (tid == 0) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w);
        for (int s = 0; s < GST; ++s) {
            mbar_init(bar(G_FULL + s), 1);
            mbar_init(bar(G_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(G_AFULL + b), 1);
            mbar_init(bar(G_AEMPTY + b), 4);  // one arrival per epilogue warp
        }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(base + G_TMEM_SLOT, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(gbase + G_TMEM_SLOT);

    const int tiles_m = cdiv(p.M, GBM), tiles_n = p.N / GBN, tiles = tiles_m * tiles_n, nk = p.K / GBK;
    constexpr uint32_t IDESC = idesc_bf16_f32(GBM, GBN, false, false);

    if (warp == 0) {
        // ================= TMA producer
        int stage = 0;
        uint32_t phase = 0, filled = 0, lastph = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            int tm, tn;
            tile_coords(t, tiles_m, tiles_n, tm, tn);
            for (int kb = 0; kb < nk; ++kb) {
                if (!gwait(bar(G_EMPTY + stage), phase ^ 1, abort)) { ok = false; break; }
                filled |= 1u << stage;
                lastph = (lastph & ~(1u << stage)) | (phase << stage);
                if (lane == 0) {
                    const uint32_t a = base + stage * GSTAGE, b = bar(G_FULL + stage);
                    mbar_expect_tx(b, GSTAGE);
                    tma_load_2d(a, &tm_x, b, kb * GBK, tm * GBM);
                    tma_load_2d(a + A_TILE, &tm_w, b, kb * GBK, tn * GBN);
                }
                __syncwarp();
                if (++stage == GST) { stage = 0; phase ^= 1; }
            }
        }
        // nothing in flight when the CTA ends
        for (int s = 0; s < GST; ++s)
            if ((filled >> s) & 1u) mbar_wait(bar(G_FULL + s), (lastph >> s) & 1u);
        if (!ok && lane == 0) report(p.status, PREFILL_ERR_TIMEOUT);
    } else if (warp == 1) {
        // ================= MMA issuer (the whole warp runs the loop; one lane issues)
        int stage = 0, local = 0;
        uint32_t phase = 0, ph_ae = 0;  // bit b: phase of accumulator b's "empty" barrier
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++local) {
            const int b = local & 1;
            if (local >= 2) {  // the epilogue has drained this accumulator
                ok = __all_sync(0xffffffffu, gwait(bar(G_AEMPTY + b), (ph_ae >> b) & 1u, abort));
                ph_ae ^= 1u << b;
                if (!ok) break;
            }
            tc_fence_after();
            const uint32_t d = tmem + (uint32_t)b * GBN;
            for (int kb = 0; kb < nk; ++kb) {
                if (!__all_sync(0xffffffffu, gwait(bar(G_FULL + stage), phase, abort))) { ok = false; break; }
                tc_fence_after();
                const uint32_t a = base + stage * GSTAGE;
                const uint64_t da = smem_desc_sw128(a, 16, 1024), db = smem_desc_sw128(a + A_TILE, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < GBK / 16; ++kk)  // 16-element K steps: +32 bytes inside the swizzle atom
                    mma_ss_elect(d, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), IDESC, (kb | kk) != 0);
                tc_commit_elect(bar(G_EMPTY + stage));  // the stage is free once these MMAs have read it
                if (++stage == GST) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
            tc_commit_elect(bar(G_AFULL + b));  // the accumulator is complete
        }
        if (!ok && lane == 0) report(p.status, PREFILL_ERR_TIMEOUT);
        __syncwarp();
    } else {
        // ================= epilogue: warp w drains TMEM lanes 32 (w % 4) .. + 31
        const int quarter = warp & 3;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        uint32_t ph_af = 0;
        int local = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++local) {
            const int b = local & 1;
            int tm, tn;
            tile_coords(t, tiles_m, tiles_n, tm, tn);
            if (!gwait(bar(G_AFULL + b), (ph_af >> b) & 1u, abort)) { ok = false; break; }
            ph_af ^= 1u << b;
            tc_fence_after();
            const int row = tm * GBM + quarter * 32 + lane;
#pragma unroll 1
            for (int c = 0; c < GBN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tmem + (uint32_t)b * GBN + (uint32_t)c * 32 + lane_off, r);
                const int n0 = tn * GBN + c * 32;  // a 32-column slice lies inside Q, K or V
                uint16_t *dst;
                if (n0 < p.hq) {
                    dst = p.q + (size_t)row * p.hq + n0;
                } else if (n0 < p.hq + p.hkv) {
                    dst = p.k + (size_t)row * p.hkv + (n0 - p.hq);
                } else {
                    dst = p.v + (size_t)row * p.hkv + (n0 - p.hq - p.hkv);
                }
                if (row < p.M) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        d4[e] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * e]), __uint_as_float(r[8 * e + 1])),
                                           pack_bf16x2(__uint_as_float(r[8 * e + 2]), __uint_as_float(r[8 * e + 3])),
                                           pack_bf16x2(__uint_as_float(r[8 * e + 4]), __uint_as_float(r[8 * e + 5])),
                                           pack_bf16x2(__uint_as_float(r[8 * e + 6]), __uint_as_float(r[8 * e + 7])));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(G_AEMPTY + b));
        }
        if (!ok && lane == 0) report(p.status, PREFILL_ERR_TIMEOUT);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int GBN>
int launch_bn(const CUtensorMap &tm_x, const CUtensorMap &tm_w, const QkvParams &p, int sms, void *stream) {
    constexpr uint32_t smem = GLay<GBN>::G_SMEM;
    cudaError_t e = cudaFuncSetAttribute(qkv_gemm_kernel<GBN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return (int)e;
    const int tiles = cdiv(p.M, GBM) * (p.N / GBN);
    const int grid = tiles < sms ? tiles : sms;
    qkv_gemm_kernel<GBN><<<grid, GTHREADS, smem, (cudaStream_t)stream>>>(tm_x, tm_w, p);
    return (int)cudaGetLastError();
}

}  // namespace

int qkv_gemm_tile_n(int M, int N, int sms) {
    // the tile width whose tiles fill the persistent grid's waves best: the
    // work is the same, the last wave's idle CTAs are not.  Measured on the
    // 8192 x 4096 x 6144 projection: 128 x 256 tiles (10.4 waves) 1448-1469
    // TFLOP/s, 128 x 192 (13.8 waves) 1475-1503, 128 x 128 (20.8 waves) 1242
    // (twice the MMA instructions and operand reads per FLOP of the 256 tile)
    auto eff = [&](int bn) {
        const long long tiles = (long long)cdiv(M, GBM) * (N / bn);
        const long long waves = (tiles + sms - 1) / sms;
        return (double)tiles / (double)(waves * sms);
    };
    if (N % 192 == 0 && (N % 256 != 0 || eff(192) > eff(256) + 0.01)) return 192;
    return 256;
}

size_t qkv_gemm_smem_bytes(int tile_n) { return tile_n == 192 ? GLay<192>::G_SMEM : GLay<256>::G_SMEM; }

int launch_qkv_gemm(const CUtensorMap &tm_x, const CUtensorMap &tm_w, const QkvParams &p, int tile_n, void *stream) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return tile_n == 192 ? launch_bn<192>(tm_x, tm_w, p, sms, stream) : launch_bn<256>(tm_x, tm_w, p, sms, stream);
}

}  // namespace pf
