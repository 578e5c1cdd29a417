// decode.cu -- paged decode attention over the cache the prefill path writes.
//
// One new token per sequence attends to its cached prefix (read page by page
// through the block table) and to itself, and its K/V are appended to the
// cache.  hncyxsy.com/news/270449 §1.1: decode feeds only the token generated
// last; hncyxsy.com/news/227904 §1: the layer then becomes matrix-vector work
// and the step is bound by memory bandwidth, i.e. by reading the KV cache.
// The result equals a chunked prefill call with one-row chunks.
//
// Design (HBM-bound; CUDA cores, no tensor cores: a query block here has
// n_head / n_kv_head rows):
//  * work unit = (sequence, kv head, split of keys_per_unit keys); the r query
//    heads of the kv head share every K/V byte read;
//  * 64-key K and V tiles are gathered page by page with cp.async (16 bytes per
//    copy, zero fill past the end) into a 3-stage ring, rows 128-byte
//    swizzled so that both the key-parallel and the column-parallel reads
//    below are free of bank conflicts; page numbers are read one tile ahead;
//  * scores: thread = (key, quarter of head_dim), partial dots for the r heads,
//    summed per key; online softmax: warp h owns head h (running max and sum);
//    P.V: thread = (pair of columns, group of keys), r x 2 accumulators;
//  * a unit's partial (unnormalised O, max, sum) is merged by
//    decode_combine_kernel when a sequence has more than one unit.
// Every wait is a cp.async group wait on the thread's own copies, so nothing
// can wait forever.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <cstdint>

#include "../../include/prefill.h"
#include "block_rule.h"
#include "decode.h"
#include "sm100.cuh"

namespace pf {
namespace {

constexpr int DT = 64;          // keys per tile
constexpr int DTHREADS = 256;   // 8 warps
constexpr int DSTAGES = 3;
constexpr int kParts = DTHREADS / DT;  // head_dim quarters in the score phase

template <int D, int R>
struct DecLay {
    static constexpr int NCH = D / 64;               // 64-column chunks of a row
    static constexpr uint32_t CHUNK = DT * 128;      // 64 rows x 128 bytes
    static constexpr uint32_t TILE = NCH * CHUNK;    // one K or V tile
    static constexpr uint32_t STAGE = 2 * TILE;      // K then V
    static constexpr uint32_t Q = DSTAGES * STAGE;   // fp32 [R][D]
    static constexpr uint32_t SPART = Q + R * D * 4; // fp32 [kParts][DT][R]
    static constexpr uint32_t P = SPART + kParts * DT * R * 4;  // fp32 [DT][8]
    static constexpr uint32_t ALPHA = P + DT * 8 * 4;           // fp32 [8]
    static constexpr uint32_t ML = ALPHA + 8 * 4;               // fp32 [8][2]
    static constexpr uint32_t BYTES = ML + 8 * 2 * 4;
    // the final reduction over key groups reuses the ring
    static constexpr int KG = DTHREADS / (D / 2);               // key groups in P.V
    static_assert((uint32_t)KG * R * D * 4 <= DSTAGES * STAGE, "reduction buffer must fit the ring");
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// byte offset of 16-byte slot `s` (0 .. D/8-1) of row `r` inside a K or V tile
template <int D>
__device__ __forceinline__ uint32_t slot_off(int r, int s) {
    return (uint32_t)(s >> 3) * (DT * 128) + (uint32_t)r * 128 + (uint32_t)(((s & 7) ^ (r & 7)) << 4);
}

template <int D, int R>
__global__ void __launch_bounds__(DTHREADS, 2) paged_decode_kernel(const DecodeParams p) {
    using L = DecLay<D, R>;
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, g = blockIdx.y, i = blockIdx.z;

    const int ctx = p.context_lens[i];
    if (ctx < 0 || ctx > p.max_ctx || (long long)ctx + 1 > (long long)p.mbps * p.block_size) {
        if (split == 0 && g == 0 && tid == 0) report(p.status, PREFILL_ERR_SHAPE);
        return;
    }
    const int nkeys = ctx + 1;  // the cached prefix and the new token
    const int nunits = cdiv(nkeys, p.keys_per_unit);
    if (split >= nunits) return;
    const int k0 = split * p.keys_per_unit;
    const int k1 = min(k0 + p.keys_per_unit, nkeys);
    const int ntiles = cdiv(k1 - k0, DT);
    const int bs = p.block_size;
    const int32_t *bt = p.block_table + (size_t)i * p.mbps;
    const size_t G = p.n_kv_head;
    const uint16_t *knew = p.k + ((size_t)i * G + g) * D;
    const uint16_t *vnew = p.v + ((size_t)i * G + g) * D;

    // the new token's K/V go to its slot (position ctx) in the last unit; no
    // unit of this call reads that slot from the cache (it reads the inputs)
    if (split == nunits - 1 && tid < 2 * (D / 8)) {
        const int page = bt[ctx / bs];
        if (page >= 0 && page < p.num_blocks) {
            const int t = tid / (D / 8), s = tid % (D / 8);
            const uint4 val = reinterpret_cast<const uint4 *>(t ? vnew : knew)[s];
            uint16_t *dst = p.cache + ((((size_t)page * 2 + t) * bs + ctx % bs) * G + g) * D;
            reinterpret_cast<uint4 *>(dst)[s] = val;
        } else {
            report(p.status, PREFILL_ERR_BLOCK_TABLE);
        }
    }

    // queries of the r heads of this kv head, fp32
    float *sq = reinterpret_cast<float *>(smem + L::Q);
    for (int x = tid; x < R * D; x += DTHREADS) {
        const int h = x / D, d = x % D;
        const uint16_t b = p.q[((size_t)i * p.n_head + (size_t)g * R + h) * D + d];
        sq[x] = __uint_as_float((uint32_t)b << 16);
    }

    // ---- loads: thread -> row tid / 4 of the tile, D/32 slots of K and of V
    constexpr int SPT = D / 32;  // slots per thread per tensor
    const int lrow = tid >> 2, lq = tid & 3;
    auto row_page = [&](int tile) -> int {  // page of this thread's row (or -1: not from the cache)
        const int pos = k0 + tile * DT + lrow;
        if (pos >= k1 || pos >= ctx) return -1;
        return __ldg(&bt[pos / bs]);
    };
    auto issue = [&](int tile, int page) {
        if (tile < ntiles) {
            const int pos = k0 + tile * DT + lrow;
            const uint32_t st = sbase + (uint32_t)(tile % DSTAGES) * L::STAGE;
            const uint16_t *src[2] = {knew, vnew};
            uint32_t bytes = 0;
            if (pos < k1) {
                if (pos == ctx) {
                    bytes = 16;  // the new token: from the inputs
                } else if (page >= 0 && page < p.num_blocks) {
                    bytes = 16;
                    src[0] = p.cache + ((((size_t)page * 2 + 0) * bs + pos % bs) * G + g) * D;
                    src[1] = p.cache + ((((size_t)page * 2 + 1) * bs + pos % bs) * G + g) * D;
                } else {
                    report(p.status, PREFILL_ERR_BLOCK_TABLE);  // zero fill
                }
            }
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int j = 0; j < SPT; ++j) {
                    const int s = lq * SPT + j;
                    cp_async16(st + t * L::TILE + slot_off<D>(lrow, s), src[t] + s * 8, bytes);
                }
        }
        cp_async_commit();  // one group per tile slot, empty past the end
    };
    int pg_next = row_page(0);
    for (int tile = 0; tile < DSTAGES - 1; ++tile) {
        const int pg = pg_next;
        pg_next = row_page(tile + 1);
        issue(tile, pg);
    }

    const float sl2 = p.scale_log2;
    float m_run = -CUDART_INF_F, l_run = 0.f;  // head `warp` (warps < R)
    // P.V accumulators: columns 2*cp, 2*cp+1 for keys kg*KPG .. of each tile
    constexpr int CP = D / 2, KPG = DT / L::KG;
    const int cp = tid % CP, kg = tid / CP;
    float acc[R][2];
#pragma unroll
    for (int h = 0; h < R; ++h) acc[h][0] = acc[h][1] = 0.f;
    float *spart = reinterpret_cast<float *>(smem + L::SPART);
    float *sp = reinterpret_cast<float *>(smem + L::P);
    float *salpha = reinterpret_cast<float *>(smem + L::ALPHA);

#pragma unroll 1
    for (int tile = 0; tile < ntiles; ++tile) {
        {
            const int pg = pg_next;
            pg_next = row_page(tile + DSTAGES);
            issue(tile + DSTAGES - 1, pg);
        }
        cp_async_wait<DSTAGES - 1>();
        __syncthreads();  // tile `tile` has landed for every thread
        const uint8_t *st = smem + (uint32_t)(tile % DSTAGES) * L::STAGE;

        // ---- scores: key kr, head_dim part pt
        {
            const int kr = tid % DT, pt = tid / DT;
            float dot[R];
#pragma unroll
            for (int h = 0; h < R; ++h) dot[h] = 0.f;
#pragma unroll
            for (int j = 0; j < D / 32; ++j) {
                const int s = pt * (D / 32) + j;
                const uint4 kv = *reinterpret_cast<const uint4 *>(st + slot_off<D>(kr, s));
                const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
                float kf[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    kf[2 * e] = __uint_as_float(w[e] << 16);
                    kf[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                }
#pragma unroll
                for (int h = 0; h < R; ++h) {
                    const float4 qa = *reinterpret_cast<const float4 *>(sq + h * D + s * 8);
                    const float4 qb = *reinterpret_cast<const float4 *>(sq + h * D + s * 8 + 4);
                    dot[h] += qa.x * kf[0] + qa.y * kf[1] + qa.z * kf[2] + qa.w * kf[3] + qb.x * kf[4] +
                              qb.y * kf[5] + qb.z * kf[6] + qb.w * kf[7];
                }
            }
#pragma unroll
            for (int h = 0; h < R; ++h) spart[(pt * DT + kr) * R + h] = dot[h];
        }
        __syncthreads();

        // ---- online softmax: warp h owns head h; lane covers keys lane, lane + 32
        if (warp < R) {
            const int h = warp;
            const int nvalid = min(DT, k1 - (k0 + tile * DT));
            float s2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int kr = lane + 32 * u;
                float s = 0.f;
#pragma unroll
                for (int pt = 0; pt < kParts; ++pt) s += spart[(pt * DT + kr) * R + h];
                s2[u] = kr < nvalid ? s : -CUDART_INF_F;
            }
            float mt = fmaxf(s2[0], s2[1]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
            const float m_new = fmaxf(m_run, mt);  // finite: every tile holds a valid key
            const float alpha = ex2((m_run - m_new) * sl2);
            const float p0 = ex2((s2[0] - m_new) * sl2), p1 = ex2((s2[1] - m_new) * sl2);
            float sum = p0 + p1;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            l_run = l_run * alpha + sum;
            m_run = m_new;
            sp[lane * 8 + h] = p0;
            sp[(lane + 32) * 8 + h] = p1;
            if (lane == 0) salpha[h] = alpha;
        }
        __syncthreads();

        // ---- O = alpha O + P V over this thread's keys and column pair
        {
#pragma unroll
            for (int h = 0; h < R; ++h) {
                const float a = salpha[h];
                acc[h][0] *= a;
                acc[h][1] *= a;
            }
            const int d = 2 * cp;
            const uint8_t *vt = st + L::TILE;
#pragma unroll
            for (int kk = 0; kk < KPG; ++kk) {
                const int kr = kg * KPG + kk;
                const uint32_t v2 =
                    *reinterpret_cast<const uint32_t *>(vt + slot_off<D>(kr, d >> 3) + (d & 7) * 2);
                const float vx = __uint_as_float(v2 << 16), vy = __uint_as_float(v2 & 0xffff0000u);
                const float4 pa = *reinterpret_cast<const float4 *>(sp + kr * 8);
                const float4 pb = *reinterpret_cast<const float4 *>(sp + kr * 8 + 4);
                const float pk[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
                for (int h = 0; h < R; ++h) {
                    acc[h][0] += pk[h] * vx;
                    acc[h][1] += pk[h] * vy;
                }
            }
        }
        __syncthreads();  // the stage and P are free for the next tile
    }
    cp_async_wait<0>();

    // ---- reduce the key groups, then write the output or this unit's partial
    float *red = reinterpret_cast<float *>(smem);  // [KG][R][D], over the drained ring
    float *sml = reinterpret_cast<float *>(smem + L::ML);
#pragma unroll
    for (int h = 0; h < R; ++h) {
        red[(kg * R + h) * D + 2 * cp] = acc[h][0];
        red[(kg * R + h) * D + 2 * cp + 1] = acc[h][1];
    }
    if (warp < R && lane == 0) {
        sml[2 * warp] = m_run * sl2;
        sml[2 * warp + 1] = l_run;
    }
    __syncthreads();
    const bool whole = nunits == 1;
    for (int x = tid; x < R * D / 2; x += DTHREADS) {  // column pairs
        const int h = x / (D / 2), d = 2 * (x % (D / 2));
        float o0 = 0.f, o1 = 0.f;
#pragma unroll
        for (int q = 0; q < L::KG; ++q) {
            o0 += red[(q * R + h) * D + d];
            o1 += red[(q * R + h) * D + d + 1];
        }
        const size_t row = (size_t)i * p.n_head + (size_t)g * R + h;
        if (whole) {
            const float inv = 1.f / sml[2 * h + 1];
            *reinterpret_cast<uint32_t *>(p.out + row * D + d) = pack_bf16x2(o0 * inv, o1 * inv);
        } else {
            const size_t prow = (size_t)split * p.num_seqs * p.n_head + row;  // [unit][seq][head]
            *reinterpret_cast<float2 *>(p.part_o + prow * D + d) = make_float2(o0, o1);
            if (d == 0) *reinterpret_cast<float2 *>(p.part_ml + prow * 2) = make_float2(sml[2 * h], sml[2 * h + 1]);
        }
    }
}

// Merge of a sequence's units: one warp per (sequence, query head), the
// online-softmax merge rule over the units' (max, sum, O).
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
    const int i = blockIdx.x;
    const int h = blockIdx.y * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (h >= p.n_head) return;
    const int ctx = p.context_lens[i];
    if (ctx < 0 || ctx > p.max_ctx || (long long)ctx + 1 > (long long)p.mbps * p.block_size) return;
    const int nunits = cdiv(ctx + 1, p.keys_per_unit);
    if (nunits <= 1) return;  // written by the unit itself
    constexpr int E = D / 32;
    const size_t row = (size_t)i * p.n_head + h;
    const size_t sstride = (size_t)p.num_seqs * p.n_head;
    float M = -CUDART_INF_F, Lsum = 0.f, acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    for (int s = 0; s < nunits; ++s) {
        const size_t prow = s * sstride + row;
        const float m = p.part_ml[prow * 2], l = p.part_ml[prow * 2 + 1];
        const float Mn = fmaxf(M, m);
        const float a = ex2(M - Mn), b = ex2(m - Mn);
        Lsum = Lsum * a + l * b;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = acc[e] * a + b * p.part_o[prow * D + lane * E + e];
        M = Mn;
    }
    const float inv = 1.f / Lsum;
    uint16_t *dst = p.out + row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 2) *reinterpret_cast<uint32_t *>(dst + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
}

template <int D, int R>
int launch_r(const DecodeParams &p, void *stream) {
    using L = DecLay<D, R>;
    const size_t smem = L::BYTES;
    cudaError_t e = cudaFuncSetAttribute(paged_decode_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return (int)e;
    dim3 grid((unsigned)p.max_units, (unsigned)p.n_kv_head, (unsigned)p.num_seqs);
    paged_decode_kernel<D, R><<<grid, DTHREADS, smem, (cudaStream_t)stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess || p.max_units <= 1) return (int)e;
    dim3 cgrid((unsigned)p.num_seqs, (unsigned)cdiv(p.n_head, 4));
    decode_combine_kernel<D><<<cgrid, 128, 0, (cudaStream_t)stream>>>(p);
    return (int)cudaGetLastError();
}

template <int D>
int launch_d(const DecodeParams &p, void *stream) {
    switch (p.n_head / p.n_kv_head) {
        case 1: return launch_r<D, 1>(p, stream);
        case 2: return launch_r<D, 2>(p, stream);
        case 3: return launch_r<D, 3>(p, stream);
        case 4: return launch_r<D, 4>(p, stream);
        case 5: return launch_r<D, 5>(p, stream);
        case 6: return launch_r<D, 6>(p, stream);
        case 7: return launch_r<D, 7>(p, stream);
        default: return launch_r<D, 8>(p, stream);
    }
}

}  // namespace

int decode_keys_per_unit(int max_ctx) {
    // units of 512 keys, fewer and longer for very long contexts (at most 64 per sequence)
    int u = 512;
    while (cdiv(max_ctx + 1, u) > kDecodeMaxUnits) u *= 2;
    return u;
}

int launch_decode(const DecodeParams &p, int head_dim, void *stream) {
    if (head_dim == 64) return launch_d<64>(p, stream);
    return launch_d<128>(p, stream);
}

}  // namespace pf
