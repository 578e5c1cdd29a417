// decode.cu -- paged decode attention over the cache the prefill path writes.
//
// One new token per sequence attends to its cached prefix (read page by page
// through the block table) and to itself, and its K/V are appended to the
// cache.  hncyxsy.com/news/270449 §1.1: decode feeds only the token generated
// last; hncyxsy.com/news/227904 §1: the layer then becomes matrix-vector work
// and the step is bound by memory bandwidth, i.e. by reading the KV cache.
// The result equals a chunked prefill call with one-row chunks.
//
// Design (HBM-bound):
//  * work unit = (sequence, kv head, split of keys_per_unit keys); the r <= 16
//    query heads of the kv head share every K/V byte read;
//  * every warp is an independent persistent worker: it takes the call's units
//    round robin (numbered densely through an exclusive scan of the units per
//    sequence, so every warp gets the same number of keys within one unit) and
//    streams them, 16 keys per step, through its own 3-stage ring
//    (cp.async, 16 bytes per copy, zero fill past the end), across unit
//    boundaries, so its loads never stop between units; a step lies in one
//    cache page (pages hold a multiple of 16 tokens), so one page-table read
//    per step, made one step ahead.  No CTA-wide barrier after the start;
//  * Q K^T and P V on warp-level tensor-core MMAs (m16n8k16, bf16 in, fp32
//    out): the query heads are the 16 rows of the A operand, the scores'
//    accumulators are the A operand of P V without leaving registers, O stays
//    in registers (16 rows x head_dim over the warp).  Rows >= r are zero
//    queries and never written out.  The running max moves only when a block
//    max exceeds it by 2^8 (as in the prefill kernel), so O is rarely rescaled;
//  * a unit's partial (unnormalised O, max, sum) is merged by
//    decode_combine_kernel when a sequence has more than one unit;
//  * FP8 mode (kFp8): the cache holds e4m3 codes with a scale per kv head;
//    the ring holds code rows and the codes are widened to f16 inside the MMA
//    fragments (see the Q K^T and P V steps), the scales folded into the
//    scores and the output; kv_store_fp8_kernel quantizes rows into the cache
//    (and, for a chunked prefill over the FP8 cache, into a dense copy of the
//    chunk's codes that the prefill kernel loads its own tiles from).
// Earlier versions for the record: CUDA-core dot products (one FMA per
// element) issued ~6.5k warp instructions per 64 keys and reached 19 % of the
// DRAM bandwidth; a CTA-wide version with tensor-core MMAs and three barriers
// per 64-key tile reached 33 %.
// Every wait is a cp.async group wait on the warp's own copies, so nothing can
// wait forever.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <cstdint>
#include <type_traits>

#include "../../include/prefill.h"
#include "block_rule.h"
#include "decode.h"
#include "sm100.cuh"

namespace pf {
namespace {

constexpr int KS = 16;            // keys per step
constexpr int WARPS = 4;          // warps (workers) per CTA
constexpr int DTHREADS = 32 * WARPS;
constexpr int NSTAGE = 3;         // ring stages per warp
constexpr int kCtasPerSm = 2;
constexpr float kLazyLog2 = 8.0f; // the running max moves when exceeded by 2^8

template <int D, bool kFp8>
struct DecLay {
    static constexpr uint32_t CHUNK = KS * 128;          // 16 rows x 128 bytes (64 columns)
    static constexpr uint32_t TILE = (D / 64) * CHUNK;   // one K or V step tile (16-bit elements)
    static constexpr uint32_t STAGE = 2 * TILE;          // K then V
    // FP8: the ring holds code rows (16 x D bytes per tensor, 16-byte segments
    // swizzled by row, see f8_off); the MMA operands are widened from them in registers
    static constexpr uint32_t F8TILE = KS * D;
    static constexpr uint32_t RING_STAGE = kFp8 ? 2 * F8TILE : STAGE;
    static constexpr uint32_t WARP_RING = NSTAGE * RING_STAGE;
    static constexpr uint32_t CTX = WARPS * WARP_RING;   // int32 [kDecodeMaxSeqs]: context lengths
    static constexpr uint32_t CUM = CTX + kDecodeMaxSeqs * 4;  // int32 [kDecodeMaxSeqs + 1]: units before sequence i
    static constexpr uint32_t BYTES = CUM + (kDecodeMaxSeqs + 1) * 4;
    static_assert(kCtasPerSm * (BYTES + 1024) <= 228 * 1024, "the resident CTAs must fit the SM");
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// D (16x8 fp32) += A (16x16, row-major fragment) x B (16x8, column fragment):
// bf16 operands, or f16 operands in the FP8 mode
template <bool kF16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (kF16) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}
// four e4m3 codes (bytes 0-3 of w) -> two f16 pairs, exact (f16 holds every
// e4m3 value): lo = (byte 0, byte 1), hi = (byte 2, byte 3), the lower byte in
// the lower half; the word's 16-bit halves go to the conversions directly
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t &lo, uint32_t &hi) {
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// byte offset of 16-byte slot `s` (0 .. D/8-1) of row `r` (0 .. 15) in a step tile:
// 64-column chunks of 16 rows x 128 bytes, slots swizzled by row
__device__ __forceinline__ uint32_t slot_off(int r, int s) {
    return (uint32_t)(s >> 3) * (KS * 128) + (uint32_t)r * 128 + (uint32_t)(((s & 7) ^ (r & 7)) << 4);
}

// byte offset of 16-byte segment `s` (0 .. D/16-1) of code row `r` in an FP8
// step tile: rows of D bytes, segments swizzled by row so that the 8 rows an
// ldmatrix reads at one segment fall in distinct banks
template <int D>
__device__ __forceinline__ uint32_t f8_off(int r, int s) {
    return (uint32_t)(r * D) + (uint32_t)((s ^ (r & (D / 16 - 1))) << 4);
}

// A work unit: keys [k0, k1) of sequence i for kv head g (split `split` of
// the sequence's nunits).  Units are numbered densely, sequence by sequence
// (then kv head, then split): unit u of the call.
struct Unit {
    int u, i, g, split, nunits, ctx, k0, k1, nsteps;
};

// Unit u (below `total`), found by binary search over the per-sequence
// cumulative unit counts; false past the end.
__device__ __forceinline__ bool get_unit(const DecodeParams &p, const int *sctx, const int *scum, int u, int total,
                                         Unit &o) {
    if (u >= total) return false;
    int lo = 0, hi = p.num_seqs - 1;  // last sequence with scum[i] <= u
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (scum[mid] <= u) lo = mid; else hi = mid - 1;
    }
    const int i = lo, ctx = sctx[i];
    const int nunits = cdiv(ctx + 1, p.keys_per_unit);  // the cached prefix and the new token
    const int rem = u - scum[i];
    o.u = u;
    o.i = i;
    o.g = rem / nunits;
    o.split = rem - o.g * nunits;
    o.nunits = nunits;
    o.ctx = ctx;
    o.k0 = o.split * p.keys_per_unit;
    o.k1 = min(o.k0 + p.keys_per_unit, ctx + 1);
    o.nsteps = cdiv(o.k1 - o.k0, KS);
    return true;
}

template <int D, bool kFp8>
__global__ void __launch_bounds__(DTHREADS, kCtasPerSm) paged_decode_kernel(const DecodeParams p) {
    using L = DecLay<D, kFp8>;
    constexpr int KSTEPS = D / 16;  // 16-column steps of Q K^T
    constexpr int NT = D / 8;       // 8-column output tiles
    extern __shared__ __align__(128) uint8_t smem[];
    // a programmatic dependent launch: the kernels before it on the stream (which
    // wrote the cache and the inputs) are complete from here on; nothing above
    // this line reads global memory
    griddep_wait();
    griddep_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t ring = smem_u32(smem) + (uint32_t)warp * L::WARP_RING;
    const int W = gridDim.x * WARPS, worker = blockIdx.x * WARPS + warp;
    const int bs = p.block_size, r = p.n_head / p.n_kv_head;
    const size_t G = p.n_kv_head;

    // context lengths and an exclusive scan of the units per sequence (n_kv_head
    // per key split; none for a sequence whose context is out of range, which
    // is skipped and reported)
    int *sctx = reinterpret_cast<int *>(smem + L::CTX);
    int *scum = reinterpret_cast<int *>(smem + L::CUM);
    __shared__ int s_wsum[WARPS];
    {
        constexpr int PER = kDecodeMaxSeqs / DTHREADS;  // sequences per thread
        int cnt[PER], run = 0;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int i = tid * PER + e;
            int c = 0;
            if (i < p.num_seqs) {
                const int ctx = __ldg(&p.context_lens[i]);
                sctx[i] = ctx;
                if (ctx < 0 || ctx > p.max_ctx || (long long)ctx + 1 > (long long)p.mbps * p.block_size) {
                    if (blockIdx.x == 0) report(p.status, PREFILL_ERR_SHAPE);
                } else {
                    c = cdiv(ctx + 1, p.keys_per_unit) * p.n_kv_head;
                }
            }
            cnt[e] = run;
            run += c;
        }
        int incl = run;  // inclusive scan of the per-thread totals over the warp
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) s_wsum[warp] = incl;
        __syncthreads();
        int base = incl - run;
        for (int w2 = 0; w2 < warp; ++w2) base += s_wsum[w2];
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int i = tid * PER + e;
            if (i <= p.num_seqs) scum[i] = base + cnt[e];  // scum[num_seqs] = total
        }
        if (tid == DTHREADS - 1 && p.num_seqs == kDecodeMaxSeqs) scum[kDecodeMaxSeqs] = base + run;
    }
    __syncthreads();  // the last CTA-wide barrier
    const int total = scum[p.num_seqs];

    // ---- load side of this warp: step (ui, si); in each copy instruction the
    // lanes fetch consecutive 16-byte slots of the step's rows
    Unit ui;
    bool has_i = get_unit(p, sctx, scum, worker, total, ui);
    int si = 0, issued = 0;
    auto step_page = [&]() -> int {  // the page holding step (ui, si) (the whole step lies in it)
        if (!has_i) return -1;
        const int pos = ui.k0 + si * KS;
        return pos < ui.ctx ? __ldg(&p.block_table[(size_t)ui.i * p.mbps + pos / bs]) : -1;
    };
    int pg_next = step_page();
    auto issue_next = [&]() {
        if (has_i) {
            const uint32_t st = ring + (uint32_t)(issued % NSTAGE) * L::RING_STAGE;
            if constexpr (kFp8) {
                // code rows: D / 16 pieces of 16 bytes per row; the new token's row
                // is zero here and written (quantized) by the compute side
                constexpr int PPR = D / 16, RPI8 = 32 / PPR;
                const int lrow = lane / PPR, s16 = lane % PPR;
                const int p0 = ui.k0 + si * KS;
                const int ncache = min(ui.k1, ui.ctx) - p0;
                const bool page_ok = pg_next >= 0 && pg_next < p.num_blocks;
                const size_t rstride = G * D;  // bytes between consecutive positions of a page
                const uint8_t *krow0 =
                    page_ok ? p.cache8 + (((size_t)pg_next * 2 * bs + p0 % bs) * G + ui.g) * D + s16 * 16 : p.cache8;
                const size_t vhalf = (size_t)bs * rstride;
#pragma unroll
                for (int j = 0; j < KS / RPI8; ++j) {
                    const int row = j * RPI8 + lrow;
                    const uint8_t *sk = p.cache8;
                    uint32_t bytes = 0;
                    if (row < ncache) {
                        if (page_ok) {
                            sk = krow0 + (size_t)row * rstride;
                            bytes = 16;
                        } else if (s16 == 0) {
                            report(p.status, PREFILL_ERR_BLOCK_TABLE);  // zero fill
                        }
                    }
                    cp_async16(st + f8_off<D>(row, s16), sk, bytes);
                    cp_async16(st + L::F8TILE + f8_off<D>(row, s16), bytes ? sk + vhalf : sk, bytes);
                }
            } else {
            constexpr int SPR = D / 8;      // 16-byte slots per row
            constexpr int RPI = 32 / SPR;   // rows per copy instruction
            const int lrow = lane / SPR, s = lane % SPR;
            const int p0 = ui.k0 + si * KS;                  // first position of the step
            const int ncache = min(ui.k1, ui.ctx) - p0;      // rows [0, ncache) come from the cache page
            const bool page_ok = pg_next >= 0 && pg_next < p.num_blocks;
            const size_t rstride = G * D;                    // elements between consecutive positions of a page
            const uint16_t *knew = p.k + ((size_t)ui.i * G + ui.g) * D + s * 8;
            const uint16_t *vnew = p.v + ((size_t)ui.i * G + ui.g) * D + s * 8;
            // row 0 of the step in the page's K half (the V half is bs positions later)
            const uint16_t *krow0 =
                page_ok ? p.cache + (((size_t)pg_next * 2 * bs + p0 % bs) * G + ui.g) * D + s * 8 : knew;
            const size_t vhalf = (size_t)bs * rstride;
            if (page_ok && ncache >= KS) {  // the common step: all 16 rows from the page
#pragma unroll
                for (int j = 0; j < KS / RPI; ++j) {
                    const int row = j * RPI + lrow;
                    const uint16_t *sk = krow0 + (size_t)row * rstride;
                    cp_async16(st + slot_off(row, s), sk, 16);
                    cp_async16(st + L::TILE + slot_off(row, s), sk + vhalf, 16);
                }
            } else {  // the new token's step or a unit's tail: per-row sources, zero fill past the end
#pragma unroll
                for (int j = 0; j < KS / RPI; ++j) {
                    const int row = j * RPI + lrow;
                    const uint16_t *sk = knew, *sv = vnew;
                    uint32_t bytes = 0;
                    if (row < ncache) {
                        if (page_ok) {
                            sk = krow0 + (size_t)row * rstride;
                            sv = sk + vhalf;
                            bytes = 16;
                        } else if (s == 0) {
                            report(p.status, PREFILL_ERR_BLOCK_TABLE);  // zero fill
                        }
                    } else if (p0 + row == ui.ctx) {
                        bytes = 16;  // the new token: from the inputs
                    }
                    cp_async16(st + slot_off(row, s), sk, bytes);
                    cp_async16(st + L::TILE + slot_off(row, s), sv, bytes);
                }
            }
            }
            ++issued;
            if (++si == ui.nsteps) {
                has_i = get_unit(p, sctx, scum, ui.u + W, total, ui);
                si = 0;
            }
            pg_next = step_page();  // read one step ahead of its use
        }
        cp_async_commit();  // one group per compute step, empty once the stream has ended
    };

    // ---- compute side: queries as A fragments in registers (rows = heads)
    const int row0 = lane >> 2, row1 = row0 + 8, c2 = 2 * (lane & 3);
    auto load_q = [&](const Unit &u, uint32_t (&qa)[KSTEPS][4]) {
        const uint32_t *q0 = reinterpret_cast<const uint32_t *>(p.q + ((size_t)u.i * p.n_head + (size_t)u.g * r) * D);
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            // FP8 mode: the 16 columns of a step are permuted (MMA k slots 2j, 2j+1,
            // 2j+8, 2j+9 <- columns 4j .. 4j+3) to match the K codes' order in the
            // widened fragments; the dot product does not depend on the order
            const int c = kFp8 ? kk * 16 + 2 * c2 : kk * 16 + c2;
            const int c_hi = kFp8 ? c + 2 : c + 8;
            qa[kk][0] = row0 < r ? __ldg(q0 + (row0 * D + c) / 2) : 0u;
            qa[kk][1] = row1 < r ? __ldg(q0 + (row1 * D + c) / 2) : 0u;
            qa[kk][2] = row0 < r ? __ldg(q0 + (row0 * D + c_hi) / 2) : 0u;
            qa[kk][3] = row1 < r ? __ldg(q0 + (row1 * D + c_hi) / 2) : 0u;
            if constexpr (kFp8) {  // bf16 pairs -> f16 pairs (exact for |q| in f16's normal range)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    qa[kk][e] = pack_f16x2(__uint_as_float(qa[kk][e] << 16), __uint_as_float(qa[kk][e] & 0xffff0000u));
            }
        }
    };
    Unit uc;
    bool has_c = get_unit(p, sctx, scum, worker, total, uc);
    int sc = 0, computed = 0;
    uint32_t qa[KSTEPS][4], qn[KSTEPS][4];
    if (has_c) load_q(uc, qa);

    const float sl2_base = p.scale_log2;
    float m_ref[2] = {-CUDART_INF_F, -CUDART_INF_F};  // rows row0, row1
    float l_part[2] = {0.f, 0.f};                       // this lane's share of the row sums
    float o[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

    for (int k = 0; k < NSTAGE - 1; ++k) issue_next();

#pragma unroll 1
    while (has_c) {
        // the FP8 codes' scales fold into the scores (K) and the output (V)
        const float sl2 = kFp8 ? sl2_base * __ldg(&p.k_scale[uc.g]) : sl2_base, thr = kLazyLog2 / sl2;
        cp_async_wait<NSTAGE - 2>();  // this step's copies (the oldest group) are done ...
        __syncwarp();                 // ... for every lane, and the previous step is finished
        issue_next();                 // into the stage the previous step used
        uint32_t st;
        if constexpr (kFp8) {
            const uint32_t f8 = ring + (uint32_t)(computed % NSTAGE) * L::RING_STAGE;
            uint8_t *f8p = smem + (f8 - smem_u32(smem));
            const int p0 = uc.k0 + sc * KS;
            if (uc.ctx >= p0 && uc.ctx < p0 + KS) {
                // the new token: quantize its K/V into the step's row and into its cache slot
                const int row = uc.ctx - p0;
                const int page = __ldg(&p.block_table[(size_t)uc.i * p.mbps + uc.ctx / bs]);
                const bool page_ok = page >= 0 && page < p.num_blocks;
                if (!page_ok && lane == 0) report(p.status, PREFILL_ERR_BLOCK_TABLE);
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const uint16_t *src = (t ? p.v : p.k) + ((size_t)uc.i * G + uc.g) * D;
                    const float sc_t = __ldg(&(t ? p.v_scale : p.k_scale)[uc.g]);
                    for (int e = lane * 4; e < D; e += 128) {  // 4 codes per lane
                        const uint2 x = __ldg(reinterpret_cast<const uint2 *>(src + e));
                        const uint32_t c01 = quant_e4m3x2(__uint_as_float(x.x << 16), __uint_as_float(x.x & 0xffff0000u), sc_t);
                        const uint32_t c23 = quant_e4m3x2(__uint_as_float(x.y << 16), __uint_as_float(x.y & 0xffff0000u), sc_t);
                        const uint32_t word = c01 | (c23 << 16);
                        *reinterpret_cast<uint32_t *>(f8p + t * L::F8TILE + f8_off<D>(row, e / 16) + e % 16) = word;
                        if (page_ok)
                            *reinterpret_cast<uint32_t *>(p.cache8 + ((((size_t)page * 2 + t) * bs + uc.ctx % bs) * G + uc.g) * D + e) = word;
                    }
                }
                __syncwarp();
            }
            st = f8;
        } else {
            st = ring + (uint32_t)(computed % NSTAGE) * L::RING_STAGE;
        }
        if (!kFp8 && sc == 0 && uc.split == uc.nunits - 1 && lane < 2 * (D / 8)) {
            // the new token's K/V to its slot (position ctx); no unit reads
            // that slot from the cache (the new token comes from the inputs)
            const int page = __ldg(&p.block_table[(size_t)uc.i * p.mbps + uc.ctx / bs]);
            if (page >= 0 && page < p.num_blocks) {
                const int t = lane / (D / 8), s = lane % (D / 8);
                const uint4 val =
                    __ldg(reinterpret_cast<const uint4 *>((t ? p.v : p.k) + ((size_t)uc.i * G + uc.g) * D) + s);
                uint16_t *dst = p.cache + ((((size_t)page * 2 + t) * bs + uc.ctx % bs) * G + uc.g) * D;
                reinterpret_cast<uint4 *>(dst)[s] = val;
            } else {
                report(p.status, PREFILL_ERR_BLOCK_TABLE);
            }
        }
        if (sc == uc.nsteps - 1) {  // the unit's last step: fetch the next unit's queries
            Unit un;
            if (get_unit(p, sctx, scum, uc.u + W, total, un)) load_q(un, qn);
        }

        // ---- S = Q K^T for the step's 16 keys (two 8-key tiles)
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (kFp8) {
            // matrices: keys 0-7 / 8-15 x segments 2j, 2j+1 of the code rows; a lane
            // receives 4 consecutive codes of one key: the k slot pairs (2j, 2j+1)
            // and (2j+8, 2j+9) of the permuted order, one conversion each
            float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
            const int m = lane >> 3;
            const int kr = (m & 1) * 8 + (lane & 7);
#pragma unroll
            for (int j = 0; j < D / 32; ++j) {
                uint32_t w[4];
                ldsm_x4(st + f8_off<D>(kr, 2 * j + (m >> 1)), w);
                uint32_t f[4][2];
#pragma unroll
                for (int e = 0; e < 4; ++e) e4m3x4_to_f16x2x2(w[e], f[e][0], f[e][1]);
                mma16816<true>(s0, qa[2 * j], f[0][0], f[0][1]);
                mma16816<true>(s1, qa[2 * j], f[1][0], f[1][1]);
                mma16816<true>(t0, qa[2 * j + 1], f[2][0], f[2][1]);
                mma16816<true>(t1, qa[2 * j + 1], f[3][0], f[3][1]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                s0[e] += t0[e];
                s1[e] += t1[e];
            }
        } else {
            // four independent accumulation chains (even / odd column steps)
            float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
            const int m = lane >> 3;  // matrices: keys 0-7 / 8-15 x columns +0 / +8
            const int kr = (m >> 1) * 8 + (lane & 7);
#pragma unroll
            for (int kk = 0; kk < KSTEPS; kk += 2) {
                uint32_t kb[4], kc[4];
                ldsm_x4(st + slot_off(kr, 2 * kk + (m & 1)), kb);
                ldsm_x4(st + slot_off(kr, 2 * kk + 2 + (m & 1)), kc);
                mma16816<kFp8>(s0, qa[kk], kb[0], kb[1]);
                mma16816<kFp8>(s1, qa[kk], kb[2], kb[3]);
                mma16816<kFp8>(t0, qa[kk + 1], kc[0], kc[1]);
                mma16816<kFp8>(t1, qa[kk + 1], kc[2], kc[3]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                s0[e] += t0[e];
                s1[e] += t1[e];
            }
        }
        // columns of this lane: keys c2, c2 + 1 (tile 0) and 8 + c2, 9 + c2 (tile 1)
        const int nvalid = uc.k1 - (uc.k0 + sc * KS);
        if (c2 >= nvalid) s0[0] = s0[2] = -CUDART_INF_F;
        if (c2 + 1 >= nvalid) s0[1] = s0[3] = -CUDART_INF_F;
        if (c2 + 8 >= nvalid) s1[0] = s1[2] = -CUDART_INF_F;
        if (c2 + 9 >= nvalid) s1[1] = s1[3] = -CUDART_INF_F;
        float mx0 = fmaxf(fmaxf(s0[0], s0[1]), fmaxf(s1[0], s1[1]));
        float mx1 = fmaxf(fmaxf(s0[2], s0[3]), fmaxf(s1[2], s1[3]));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        // lazy max: move it (and rescale O and the sums) only past the threshold;
        // every step holds a valid key, so a row's first step always moves it
        const bool mv0 = mx0 > m_ref[0] + thr, mv1 = mx1 > m_ref[1] + thr;
        if (__any_sync(0xffffffffu, mv0 || mv1)) {
            const float n0 = mv0 ? mx0 : m_ref[0], n1 = mv1 ? mx1 : m_ref[1];
            const float a0 = ex2((m_ref[0] - n0) * sl2), a1 = ex2((m_ref[1] - n1) * sl2);
            m_ref[0] = n0;
            m_ref[1] = n1;
            l_part[0] *= a0;
            l_part[1] *= a1;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                o[nt][0] *= a0;
                o[nt][1] *= a0;
                o[nt][2] *= a1;
                o[nt][3] *= a1;
            }
        }
        const float nm0 = -m_ref[0] * sl2, nm1 = -m_ref[1] * sl2;
        const float p00 = ex2(fmaf(s0[0], sl2, nm0)), p01 = ex2(fmaf(s0[1], sl2, nm0));
        const float p02 = ex2(fmaf(s0[2], sl2, nm1)), p03 = ex2(fmaf(s0[3], sl2, nm1));
        const float p10 = ex2(fmaf(s1[0], sl2, nm0)), p11 = ex2(fmaf(s1[1], sl2, nm0));
        const float p12 = ex2(fmaf(s1[2], sl2, nm1)), p13 = ex2(fmaf(s1[3], sl2, nm1));
        l_part[0] += (p00 + p01) + (p10 + p11);
        l_part[1] += (p02 + p03) + (p12 + p13);
        // the scores' accumulators are the A fragment of P V (16 rows x 16 keys)
        uint32_t pa[4];
        if constexpr (kFp8) {
            pa[0] = pack_f16x2(p00, p01);
            pa[1] = pack_f16x2(p02, p03);
            pa[2] = pack_f16x2(p10, p11);
            pa[3] = pack_f16x2(p12, p13);
        } else {
            pa[0] = pack_bf16x2(p00, p01);
            pa[1] = pack_bf16x2(p02, p03);
            pa[2] = pack_bf16x2(p10, p11);
            pa[3] = pack_bf16x2(p12, p13);
        }

        // ---- O += P V over all output columns
        if constexpr (kFp8) {
            // transposed matrices: keys 0-7 / 8-15 x segments 2c, 2c+1; a lane receives,
            // for keys 2j and 2j+1, the codes of columns 16 seg + 2 (lane / 4) and + 1:
            // bytes 0 and 2 form the pair of the even-column tile, bytes 1 and 3 the
            // odd one.  o[4c + 2 h + e] holds segment 2c + h, column parity e.
            const int m = lane >> 3;
            const int vr = (m & 1) * 8 + (lane & 7);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t w[4];
                ldsm_x4_t(st + L::F8TILE + f8_off<D>(vr, 2 * c + (m >> 1)), w);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t lo = w[2 * h], hi = w[2 * h + 1];  // keys 0-7, keys 8-15
                    // even columns: (lo byte 0, lo byte 2 | hi byte 0, hi byte 2); odd: bytes 1, 3
                    uint32_t ev[2], od[2];
                    e4m3x4_to_f16x2x2(__byte_perm(lo, hi, 0x6420), ev[0], ev[1]);
                    e4m3x4_to_f16x2x2(__byte_perm(lo, hi, 0x7531), od[0], od[1]);
                    mma16816<true>(o[4 * c + 2 * h], pa, ev[0], ev[1]);
                    mma16816<true>(o[4 * c + 2 * h + 1], pa, od[0], od[1]);
                }
            }
        } else {
            const int m = lane >> 3;  // matrices: keys 0-7 / 8-15 x columns +0 / +8
            const int vr = (m & 1) * 8 + (lane & 7);
#pragma unroll
            for (int c = 0; c < NT / 2; ++c) {
                uint32_t vb[4];
                ldsm_x4_t(st + L::TILE + slot_off(vr, 2 * c + (m >> 1)), vb);
                mma16816<false>(o[2 * c], pa, vb[0], vb[1]);
                mma16816<false>(o[2 * c + 1], pa, vb[2], vb[3]);
            }
        }
        ++computed;
        if (++sc < uc.nsteps) continue;

        // ---- end of the unit: row sums over the 4 lanes of a row, then rows < r out
        float l0 = l_part[0], l1 = l_part[1];
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        const bool whole = uc.nunits == 1;
        const size_t hrow = (size_t)uc.i * p.n_head + (size_t)uc.g * r;
        const float vsc = kFp8 ? __ldg(&p.v_scale[uc.g]) : 1.f;  // the V codes' scale
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int h = hh ? row1 : row0;
            if (h >= r) continue;
            const float lsum = hh ? l1 : l0;
            const size_t row = hrow + h;
            if constexpr (kFp8) {
                // segment sg: this lane's columns 16 sg + 4 (lane % 4) + 0 .. 3 are the even
                // tile's two values and the odd tile's two values, interleaved
                const float f = whole ? vsc / lsum : vsc;
                const size_t prow = (size_t)uc.split * p.num_seqs * p.n_head + row;  // [unit][seq][head]
#pragma unroll
                for (int sg = 0; sg < D / 16; ++sg) {
                    const float *ev = o[4 * (sg >> 1) + 2 * (sg & 1)], *od = o[4 * (sg >> 1) + 2 * (sg & 1) + 1];
                    const float v0 = ev[2 * hh] * f, v1 = od[2 * hh] * f, v2 = ev[2 * hh + 1] * f, v3 = od[2 * hh + 1] * f;
                    const int col = 16 * sg + 2 * c2;
                    if (whole)
                        *reinterpret_cast<uint2 *>(p.out + row * D + col) = make_uint2(pack_bf16x2(v0, v1), pack_bf16x2(v2, v3));
                    else
                        *reinterpret_cast<float4 *>(p.part_o + prow * D + col) = make_float4(v0, v1, v2, v3);
                }
                if (!whole && (lane & 3) == 0)
                    *reinterpret_cast<float2 *>(p.part_ml + prow * 2) = make_float2(m_ref[hh] * sl2, lsum);
            } else if (whole) {
                const float inv = vsc / lsum;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    *reinterpret_cast<uint32_t *>(p.out + row * D + nt * 8 + c2) =
                        pack_bf16x2(o[nt][2 * hh] * inv, o[nt][2 * hh + 1] * inv);
            } else {
                const size_t prow = (size_t)uc.split * p.num_seqs * p.n_head + row;  // [unit][seq][head]
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    *reinterpret_cast<float2 *>(p.part_o + prow * D + nt * 8 + c2) =
                        make_float2(o[nt][2 * hh] * vsc, o[nt][2 * hh + 1] * vsc);
                if ((lane & 3) == 0)
                    *reinterpret_cast<float2 *>(p.part_ml + prow * 2) = make_float2(m_ref[hh] * sl2, lsum);
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
        m_ref[0] = m_ref[1] = -CUDART_INF_F;
        l_part[0] = l_part[1] = 0.f;
        has_c = get_unit(p, sctx, scum, uc.u + W, total, uc);
        sc = 0;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk)
#pragma unroll
            for (int e = 0; e < 4; ++e) qa[kk][e] = qn[kk][e];
    }
    cp_async_wait<0>();  // nothing in flight when the warp exits
}

// Merge of a sequence's units: one warp per (sequence, query head), the
// online-softmax merge rule over the units' (max, sum, O): lane s holds unit
// s's max and sum (and s + 32's), so the weights 2^(m_s - M) come from one warp
// max and one warp sum; the O rows are then summed with independent loads.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
    griddep_wait();  // the decode kernel's partials are complete (programmatic dependent launch)
    griddep_launch_dependents();
    const int i = blockIdx.x;
    const int h = blockIdx.y * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (h >= p.n_head) return;
    const int ctx = p.context_lens[i];
    if (ctx < 0 || ctx > p.max_ctx || (long long)ctx + 1 > (long long)p.mbps * p.block_size) return;
    const int nunits = cdiv(ctx + 1, p.keys_per_unit);  // <= kDecodeMaxUnits = 64
    if (nunits <= 1) return;                             // written by the unit itself
    constexpr int E = D / 32;
    const size_t row = (size_t)i * p.n_head + h;
    const size_t sstride = (size_t)p.num_seqs * p.n_head;
    float m[2], l[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int sidx = lane + 32 * u;
        m[u] = -CUDART_INF_F;
        l[u] = 0.f;
        if (sidx < nunits) {
            const float2 ml = *reinterpret_cast<const float2 *>(p.part_ml + (sidx * sstride + row) * 2);
            m[u] = ml.x;
            l[u] = ml.y;
        }
    }
    float M = fmaxf(m[0], m[1]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float w0 = ex2(m[0] - M), w1 = ex2(m[1] - M);  // 0 for absent units
    float Lsum = w0 * l[0] + w1 * l[1];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, off);
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
#pragma unroll 4
    for (int s = 0; s < nunits; ++s) {
        const float wgt = __shfl_sync(0xffffffffu, s < 32 ? w0 : w1, s & 31);
        const float *src = p.part_o + (s * sstride + row) * D + lane * E;
        if constexpr (E == 4) {
            const float4 f = *reinterpret_cast<const float4 *>(src);
            acc[0] += wgt * f.x;
            acc[1] += wgt * f.y;
            acc[2] += wgt * f.z;
            acc[3] += wgt * f.w;
        } else {
            const float2 f = *reinterpret_cast<const float2 *>(src);
            acc[0] += wgt * f.x;
            acc[1] += wgt * f.y;
        }
    }
    const float inv = 1.f / Lsum;
    uint16_t *dst = p.out + row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 2) *reinterpret_cast<uint32_t *>(dst + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
}

// ------------------------------------------------------------------ whole-page decode
// The kernel for kv-head counts that are a multiple of 8 (and, for the FP8
// cache, head_dim 128).  The cache stores a page's tokens with all kv heads of
// a token side by side ([bs][n_kv_head][D] per page half), so the 16 tokens of
// a step hold 8 kv heads' rows in one contiguous 16 x 8 x D run of each half.
// One CTA per SM takes work units (sequence, slab of 8 kv heads, key split):
//  * warp 8 (producer) TMA-loads each step's K and V for the whole slab --
//    boxes of 16 tokens x 8 heads x 128 bytes, 128-byte swizzled -- into a
//    ring of 64 KB stages (bf16, head_dim 128; 32 KB otherwise), so the DRAM
//    reads are whole contiguous page runs and one thread issues them;
//  * warps 0-7 compute, warp w the kv head 8 * slab + w, exactly as the
//    per-warp kernel does (Q K^T and P V on m16n8k16 MMAs from ldmatrix
//    fragments, lazy running max), and release the stage (count 8);
//  * the new token (position ctx, last key split) is written over its row of
//    the loaded step by the warp of its kv head, rows past it are zeroed in V
//    (their bytes are whatever the page holds), and its K/V go to the cache.
// Units, key splits and the partials' layout are those of the per-warp
// kernel, so decode_combine_kernel merges the splits of either.
constexpr int TW = 8;          // compute warps: the kv heads of a slab
constexpr int TTHREADS = 384;  // + a warpgroup whose warp 8 is the TMA producer (9-11 idle)

template <int D, bool kFp8>
struct TLay {
    static constexpr int NCH = kFp8 ? 1 : D / 64;   // 128-byte chunks of a (token, head) row
    static constexpr uint32_t HEADB = KS * 128;     // one head's 16 token rows of one chunk
    static constexpr uint32_t CHB = TW * HEADB;     // one chunk of the slab (16 KB)
    static constexpr uint32_t TILE = NCH * CHB;     // K (or V): 16 tokens x 8 heads
    static constexpr uint32_t STAGE = 2 * TILE;     // K, then V
    static constexpr int NST = (192 * 1024) / STAGE;
    static constexpr uint32_t BAR = NST * STAGE;    // full[NST], empty[NST]
    static constexpr uint32_t ABORT = BAR + 2 * NST * 8;
    static constexpr uint32_t CTX = ABORT + 16;     // int32 [kDecodeMaxSeqs]
    static constexpr uint32_t CUM = CTX + kDecodeMaxSeqs * 4;  // int32 [kDecodeMaxSeqs + 1]
    static constexpr uint32_t BYTES = CUM + (kDecodeMaxSeqs + 1) * 4;
    static_assert(!kFp8 || D == 128, "FP8 rows of D codes are one 128-byte swizzle row");
    static_assert(NST >= 3, "ring depth");
    static_assert(BYTES + 1024 <= 227 * 1024, "the CTA must fit the SM");
};

// byte offset of 16-byte slot s (0 .. 8 * NCH - 1) of token row t within one
// head's part of a tile (bf16): 64-column chunks CHB apart, slots swizzled by
// the row, as the TMA's 128-byte swizzle lays them out (1024-byte aligned
// tiles; a head's 16 rows start on a 2 KB boundary)
template <int D, bool kFp8>
__device__ __forceinline__ uint32_t tslot_off(int t, int s) {
    using L = TLay<D, kFp8>;
    return (uint32_t)(s >> 3) * L::CHB + (uint32_t)t * 128 + (uint32_t)(((s & 7) ^ (t & 7)) << 4);
}

// Work of the whole-page kernel, balanced by 16-key steps.  The call's steps
// form one list: sequence by sequence, and within a sequence slab by slab
// (segment s = i * nslab + slab holds the sequence's cdiv(ctx + 1, 16) steps for
// the kv heads of that slab).  CTA c takes steps [c T, (c + 1) T) of the list,
// T = max(kMinStepsPerCta, cdiv(S, grid)) for S steps in all, so every CTA gets
// the same number of steps whatever the context lengths.  A piece is the part
// of one segment inside one CTA's range; a segment cut by CTA boundaries has
// pieces c0 .. c1 (c0 = seg_start / T, c1 = (seg_end - 1) / T), and piece
// (c, s) has the id c + s, unique and below grid + segments (a later CTA can
// only overlap a later or the same segment), which numbers its partial rows.
constexpr int kMinStepsPerCta = 16;  // 256 keys: no finer cuts of a short call
__host__ __device__ __forceinline__ int steps_per_cta(int S, int grid) {
    const int t = (S + grid - 1) / grid;
    return t > kMinStepsPerCta ? t : kMinStepsPerCta;
}

struct TPiece {
    int i, slab, ctx, k0, k1, nsteps;  // keys [k0, k1) of sequence i, kv heads of slab
    int pid, npieces;                  // piece id (partial rows), pieces of its segment
    int gnext;                         // first list step after this piece
};
// The piece that starts at list step g (below the CTA's end gend).
__device__ __forceinline__ TPiece get_piece(const DecodeParams &p, const int *sctx, const int *scum, int nslab,
                                            int T, int cta, int g, int gend) {
    int lo = 0, hi = p.num_seqs - 1;  // last sequence with scum[i] <= g (sequences without steps are skipped)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (scum[mid] <= g) lo = mid; else hi = mid - 1;
    }
    TPiece o;
    o.i = lo;
    o.ctx = sctx[lo];
    const int ns = cdiv(o.ctx + 1, KS);
    const int rel = g - scum[lo];
    o.slab = rel / ns;
    const int seg_start = scum[lo] + o.slab * ns, seg_end = seg_start + ns;
    const int a = g - seg_start, b = min(seg_end, gend) - seg_start;
    o.k0 = a * KS;
    o.k1 = min(b * KS, o.ctx + 1);
    o.nsteps = b - a;
    o.npieces = (seg_end - 1) / T - seg_start / T + 1;
    o.pid = cta + lo * nslab + o.slab;
    o.gnext = seg_start + b;
    return o;
}

template <int D, bool kFp8>
__global__ void __launch_bounds__(TTHREADS, 1)
paged_decode_tma_kernel(const __grid_constant__ CUtensorMap tm, const DecodeParams p) {
    using L = TLay<D, kFp8>;
    constexpr int KSTEPS = D / 16;  // 16-column steps of Q K^T
    constexpr int NT = D / 8;       // 8-column output tiles
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // 128-byte swizzle atoms: 1024-byte aligned tiles
    uint8_t *sm = smem_raw + (base - raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bs = p.block_size, r = p.n_head / p.n_kv_head;
    const size_t G = p.n_kv_head;
    const int nslab = p.n_kv_head / TW;
    volatile int *abort = reinterpret_cast<volatile int *>(sm + L::ABORT);
    auto full = [&](int s) -> uint32_t { return base + L::BAR + 8u * s; };
    auto empty = [&](int s) -> uint32_t { return base + L::BAR + 8u * (L::NST + s); };
    if (tid == 0) {
        tma_prefetch_desc(&tm);
        for (int s = 0; s < L::NST; ++s) {
            mbar_init(full(s), 1);    // the producer's expect_tx (+ the TMA bytes)
            mbar_init(empty(s), TW);  // one arrive per compute warp
        }
        *abort = 0;
        fence_mbar_init();
    }
    // a programmatic dependent launch: nothing above this line reads global memory
    griddep_wait();
    griddep_launch_dependents();

    // context lengths and an exclusive scan of the units per sequence
    int *sctx = reinterpret_cast<int *>(sm + L::CTX);
    int *scum = reinterpret_cast<int *>(sm + L::CUM);
    __shared__ int s_wsum[TTHREADS / 32];
    {
        constexpr int PER = (kDecodeMaxSeqs + TTHREADS - 1) / TTHREADS;  // covers index num_seqs too
        int cnt[PER], run = 0;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int i = tid * PER + e;
            int c = 0;
            if (i < p.num_seqs) {
                const int ctx = __ldg(&p.context_lens[i]);
                sctx[i] = ctx;
                if (ctx < 0 || ctx > p.max_ctx || (long long)ctx + 1 > (long long)p.mbps * p.block_size) {
                    if (blockIdx.x == 0) report(p.status, PREFILL_ERR_SHAPE);
                } else {
                    c = cdiv(ctx + 1, KS) * nslab;  // the sequence's steps, all slabs
                }
            }
            cnt[e] = run;
            run += c;
        }
        int incl = run;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) s_wsum[warp] = incl;
        __syncthreads();
        int base_u = incl - run;
        for (int w2 = 0; w2 < warp; ++w2) base_u += s_wsum[w2];
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int i = tid * PER + e;
            if (i <= p.num_seqs) {
                scum[i] = base_u + cnt[e];
                if (blockIdx.x == 0 && p.seg_cum) p.seg_cum[i] = base_u + cnt[e];  // for the merge kernel
            }
        }
    }
    __syncthreads();  // the last CTA-wide barrier
    const int S = scum[p.num_seqs];
    const int T = steps_per_cta(S, gridDim.x), cta = blockIdx.x;
    const int gbeg = min(cta * T, S), gend = min(gbeg + T, S);  // this CTA's steps

    // register split (384 threads x 168 at launch = 64,512): compute warpgroups
    // 2 x 128 x 224, the producer's warpgroup 128 x 56
    if (warp >= TW) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 56;");
        if (warp != TW) return;
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 224;");
    }
    if (warp == TW) {
        // ================= producer: one step = K and V of 16 tokens x 8 kv heads
        int stage = 0;
        uint32_t phase = 0, filled = 0, lastph = 0;
        bool ok = true;
        for (int g = gbeg; ok && g < gend;) {
            const TPiece u = get_piece(p, sctx, scum, nslab, T, cta, g, gend);
            g = u.gnext;
            for (int s = 0; s < u.nsteps; ++s) {
                const int p0 = u.k0 + s * KS;  // a step lies in one page (pages hold multiples of 16)
                int page = 0;
                if (lane == 0) page = __ldg(&p.block_table[(size_t)u.i * p.mbps + p0 / bs]);
                page = __shfl_sync(0xffffffffu, page, 0);
                if (page < 0 || page >= p.num_blocks) {
                    if (lane == 0) report(p.status, PREFILL_ERR_BLOCK_TABLE);
                    page = p.num_blocks;  // outside the map: the boxes read zeros
                }
                if (!mbar_wait(empty(stage), phase ^ 1u, abort)) { ok = false; break; }
                filled |= 1u << stage;
                lastph = (lastph & ~(1u << stage)) | (phase << stage);
                if (lane == 0) mbar_expect_tx(full(stage), L::STAGE);
                __syncwarp();
                if (lane < 2 * L::NCH) {  // lanes issue together: K chunks, then V chunks
                    const int t = lane / L::NCH, c = lane % L::NCH;
                    tma_load_4d(base + stage * L::STAGE + t * L::TILE + c * L::CHB, &tm, full(stage), c * 64,
                                p0 % bs, u.slab * TW, page * 2 + t);
                }
                if (++stage == L::NST) { stage = 0; phase ^= 1u; }
            }
        }
        if (!ok) {
            *abort = 1;
            if (lane == 0) report(p.status, PREFILL_ERR_TIMEOUT);
        }
        // no copy may be in flight when the CTA ends
        for (int st = 0; st < L::NST; ++st)
            if ((filled >> st) & 1u) mbar_wait(full(st), (lastph >> st) & 1u);
        return;
    }

    // ================= compute warps: warp w runs kv head 8 * slab + w of each unit
    const int row0 = lane >> 2, row1 = row0 + 8, c2 = 2 * (lane & 3);
    auto load_q = [&](int i, int g, uint32_t (&qa)[KSTEPS][4]) {
        const uint32_t *q0 = reinterpret_cast<const uint32_t *>(p.q + ((size_t)i * p.n_head + (size_t)g * r) * D);
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            // FP8: the columns of a 16-column step are permuted to the K codes'
            // order in the widened fragments (see paged_decode_kernel)
            const int c = kFp8 ? kk * 16 + 2 * c2 : kk * 16 + c2;
            const int c_hi = kFp8 ? c + 2 : c + 8;
            qa[kk][0] = row0 < r ? __ldg(q0 + (row0 * D + c) / 2) : 0u;
            qa[kk][1] = row1 < r ? __ldg(q0 + (row1 * D + c) / 2) : 0u;
            qa[kk][2] = row0 < r ? __ldg(q0 + (row0 * D + c_hi) / 2) : 0u;
            qa[kk][3] = row1 < r ? __ldg(q0 + (row1 * D + c_hi) / 2) : 0u;
            if constexpr (kFp8) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    qa[kk][e] = pack_f16x2(__uint_as_float(qa[kk][e] << 16), __uint_as_float(qa[kk][e] & 0xffff0000u));
            }
        }
    };
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    bool has = gbeg < gend;
    TPiece uc;
    if (has) uc = get_piece(p, sctx, scum, nslab, T, cta, gbeg, gend);
    uint32_t qa[KSTEPS][4], qn[KSTEPS][4];
    if (has) load_q(uc.i, uc.slab * TW + warp, qa);
#pragma unroll 1
    while (has) {
        const int g = uc.slab * TW + warp;
        const float sl2 = kFp8 ? p.scale_log2 * __ldg(&p.k_scale[g]) : p.scale_log2, thr = kLazyLog2 / sl2;
        float m_ref[2] = {-CUDART_INF_F, -CUDART_INF_F};
        float l_part[2] = {0.f, 0.f};
        float o[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
        const bool has_n = uc.gnext < gend;
        TPiece un;
        if (has_n) un = get_piece(p, sctx, scum, nslab, T, cta, uc.gnext, gend);
#pragma unroll 1
        for (int sc = 0; sc < uc.nsteps; ++sc) {
            if (!mbar_wait(full(stage), phase, abort)) { ok = false; break; }
            const uint32_t kt = base + stage * L::STAGE + warp * L::HEADB;  // this head's K rows
            const uint32_t vt = kt + L::TILE;                                // and V rows
            const int p0 = uc.k0 + sc * KS;
            if (uc.ctx >= p0 && uc.ctx < p0 + KS) {
                // the new token's step: its row comes from the inputs (and goes to
                // its cache slot); V rows past it are zeroed, since P is 0 there but
                // the page's bytes may hold anything (a NaN would survive 0 x NaN)
                const int nr = uc.ctx - p0;
                const int page = __ldg(&p.block_table[(size_t)uc.i * p.mbps + uc.ctx / bs]);
                const bool page_ok = page >= 0 && page < p.num_blocks;
                if (!page_ok && lane == 0) report(p.status, PREFILL_ERR_BLOCK_TABLE);
                if constexpr (kFp8) {
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const uint16_t *src = (t ? p.v : p.k) + ((size_t)uc.i * G + g) * D;
                        const float sc_t = __ldg(&(t ? p.v_scale : p.k_scale)[g]);
                        const int e = lane * 4;  // 4 codes per lane (D = 128)
                        const uint2 x = __ldg(reinterpret_cast<const uint2 *>(src + e));
                        const uint32_t c01 = quant_e4m3x2(__uint_as_float(x.x << 16), __uint_as_float(x.x & 0xffff0000u), sc_t);
                        const uint32_t c23 = quant_e4m3x2(__uint_as_float(x.y << 16), __uint_as_float(x.y & 0xffff0000u), sc_t);
                        const uint32_t word = c01 | (c23 << 16);
                        *reinterpret_cast<uint32_t *>(sm + ((t ? vt : kt) - base) + f8_off<D>(nr, e / 16) + e % 16) = word;
                        if (page_ok)
                            *reinterpret_cast<uint32_t *>(p.cache8 + ((((size_t)page * 2 + t) * bs + uc.ctx % bs) * G + g) * D + e) = word;
                    }
                    for (int x = lane; x < (KS - 1 - nr) * (D / 16); x += 32) {
                        const int row = nr + 1 + x / (D / 16), seg = x % (D / 16);
                        *reinterpret_cast<uint4 *>(sm + (vt - base) + f8_off<D>(row, seg)) = make_uint4(0, 0, 0, 0);
                    }
                } else {
                    constexpr int SPR = D / 8;  // 16-byte slots per row
                    if (lane < 2 * SPR) {
                        const int t = lane / SPR, s = lane % SPR;
                        const uint4 val =
                            __ldg(reinterpret_cast<const uint4 *>((t ? p.v : p.k) + ((size_t)uc.i * G + g) * D) + s);
                        *reinterpret_cast<uint4 *>(sm + ((t ? vt : kt) - base) + tslot_off<D, kFp8>(nr, s)) = val;
                        if (page_ok)
                            reinterpret_cast<uint4 *>(p.cache + ((((size_t)page * 2 + t) * bs + uc.ctx % bs) * G + g) * D)[s] = val;
                    }
                    for (int x = lane; x < (KS - 1 - nr) * SPR; x += 32) {
                        const int row = nr + 1 + x / SPR, s = x % SPR;
                        *reinterpret_cast<uint4 *>(sm + (vt - base) + tslot_off<D, kFp8>(row, s)) = make_uint4(0, 0, 0, 0);
                    }
                }
                fence_proxy_async_smem();  // these writes come before the stage's next TMA fill
                __syncwarp();
            }

            if (sc == uc.nsteps - 1 && has_n) load_q(un.i, un.slab * TW + warp, qn);  // the next unit's queries

            // ---- S = Q K^T for the step's 16 keys (two 8-key tiles)
            float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
            {
                float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
                const int m = lane >> 3;
                if constexpr (kFp8) {
                    const int kr = (m & 1) * 8 + (lane & 7);
#pragma unroll
                    for (int j = 0; j < D / 32; ++j) {
                        uint32_t w[4];
                        ldsm_x4(kt + f8_off<D>(kr, 2 * j + (m >> 1)), w);
                        uint32_t f[4][2];
#pragma unroll
                        for (int e = 0; e < 4; ++e) e4m3x4_to_f16x2x2(w[e], f[e][0], f[e][1]);
                        mma16816<true>(s0, qa[2 * j], f[0][0], f[0][1]);
                        mma16816<true>(s1, qa[2 * j], f[1][0], f[1][1]);
                        mma16816<true>(t0, qa[2 * j + 1], f[2][0], f[2][1]);
                        mma16816<true>(t1, qa[2 * j + 1], f[3][0], f[3][1]);
                    }
                } else {
                    const int kr = (m >> 1) * 8 + (lane & 7);  // matrices: keys 0-7 / 8-15 x columns +0 / +8
#pragma unroll
                    for (int kk = 0; kk < KSTEPS; kk += 2) {
                        uint32_t kb[4], kc[4];
                        ldsm_x4(kt + tslot_off<D, kFp8>(kr, 2 * kk + (m & 1)), kb);
                        ldsm_x4(kt + tslot_off<D, kFp8>(kr, 2 * kk + 2 + (m & 1)), kc);
                        mma16816<false>(s0, qa[kk], kb[0], kb[1]);
                        mma16816<false>(s1, qa[kk], kb[2], kb[3]);
                        mma16816<false>(t0, qa[kk + 1], kc[0], kc[1]);
                        mma16816<false>(t1, qa[kk + 1], kc[2], kc[3]);
                    }
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    s0[e] += t0[e];
                    s1[e] += t1[e];
                }
            }
            // FP8: the step's V codes widened to f16 fragments here -- they do not depend
            // on the scores, so their loads and conversions overlap the S products and
            // the softmax instead of following them
            uint32_t vf[kFp8 ? D / 32 : 1][2][4];
            if constexpr (kFp8) {
                const int m = lane >> 3;
                const int vr = (m & 1) * 8 + (lane & 7);
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t w[4];
                    ldsm_x4_t(vt + f8_off<D>(vr, 2 * c + (m >> 1)), w);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t lo = w[2 * h], hi = w[2 * h + 1];
                        // even columns: (lo byte 0, lo byte 2 | hi byte 0, hi byte 2); odd: bytes 1, 3
                        e4m3x4_to_f16x2x2(__byte_perm(lo, hi, 0x6420), vf[c][h][0], vf[c][h][1]);
                        e4m3x4_to_f16x2x2(__byte_perm(lo, hi, 0x7531), vf[c][h][2], vf[c][h][3]);
                    }
                }
            }
            const int nvalid = uc.k1 - p0;
            if (c2 >= nvalid) s0[0] = s0[2] = -CUDART_INF_F;
            if (c2 + 1 >= nvalid) s0[1] = s0[3] = -CUDART_INF_F;
            if (c2 + 8 >= nvalid) s1[0] = s1[2] = -CUDART_INF_F;
            if (c2 + 9 >= nvalid) s1[1] = s1[3] = -CUDART_INF_F;
            float mx0 = fmaxf(fmaxf(s0[0], s0[1]), fmaxf(s1[0], s1[1]));
            float mx1 = fmaxf(fmaxf(s0[2], s0[3]), fmaxf(s1[2], s1[3]));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const bool mv0 = mx0 > m_ref[0] + thr, mv1 = mx1 > m_ref[1] + thr;
            if (__any_sync(0xffffffffu, mv0 || mv1)) {
                const float n0 = mv0 ? mx0 : m_ref[0], n1 = mv1 ? mx1 : m_ref[1];
                const float a0 = ex2((m_ref[0] - n0) * sl2), a1 = ex2((m_ref[1] - n1) * sl2);
                m_ref[0] = n0;
                m_ref[1] = n1;
                l_part[0] *= a0;
                l_part[1] *= a1;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    o[nt][0] *= a0;
                    o[nt][1] *= a0;
                    o[nt][2] *= a1;
                    o[nt][3] *= a1;
                }
            }
            const float nm0 = -m_ref[0] * sl2, nm1 = -m_ref[1] * sl2;
            const float p00 = ex2(fmaf(s0[0], sl2, nm0)), p01 = ex2(fmaf(s0[1], sl2, nm0));
            const float p02 = ex2(fmaf(s0[2], sl2, nm1)), p03 = ex2(fmaf(s0[3], sl2, nm1));
            const float p10 = ex2(fmaf(s1[0], sl2, nm0)), p11 = ex2(fmaf(s1[1], sl2, nm0));
            const float p12 = ex2(fmaf(s1[2], sl2, nm1)), p13 = ex2(fmaf(s1[3], sl2, nm1));
            l_part[0] += (p00 + p01) + (p10 + p11);
            l_part[1] += (p02 + p03) + (p12 + p13);
            uint32_t pa[4];
            if constexpr (kFp8) {
                pa[0] = pack_f16x2(p00, p01);
                pa[1] = pack_f16x2(p02, p03);
                pa[2] = pack_f16x2(p10, p11);
                pa[3] = pack_f16x2(p12, p13);
            } else {
                pa[0] = pack_bf16x2(p00, p01);
                pa[1] = pack_bf16x2(p02, p03);
                pa[2] = pack_bf16x2(p10, p11);
                pa[3] = pack_bf16x2(p12, p13);
            }
            // ---- O += P V over all output columns
            {
                const int m = lane >> 3;
                const int vr = (m & 1) * 8 + (lane & 7);
                if constexpr (kFp8) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c)
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            mma16816<true>(o[4 * c + 2 * h], pa, vf[c][h][0], vf[c][h][1]);
                            mma16816<true>(o[4 * c + 2 * h + 1], pa, vf[c][h][2], vf[c][h][3]);
                        }
                } else {
#pragma unroll
                    for (int c = 0; c < NT / 2; ++c) {
                        uint32_t vb[4];
                        ldsm_x4_t(vt + tslot_off<D, kFp8>(vr, 2 * c + (m >> 1)), vb);
                        mma16816<false>(o[2 * c], pa, vb[0], vb[1]);
                        mma16816<false>(o[2 * c + 1], pa, vb[2], vb[3]);
                    }
                }
            }
            __syncwarp();  // every lane's reads of the stage are done
            if (lane == 0) mbar_arrive(empty(stage));
            if (++stage == L::NST) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;

        // ---- end of the unit: row sums over the 4 lanes of a row, then rows < r out
        float l0 = l_part[0], l1 = l_part[1];
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        const bool whole = uc.npieces == 1;
        const size_t hrow = (size_t)uc.i * p.n_head + (size_t)g * r;
        // partial rows of this piece: [pid][8 r heads of the slab]
        const size_t prow0 = (size_t)uc.pid * (TW * r) + (size_t)warp * r;
        const float vsc = kFp8 ? __ldg(&p.v_scale[g]) : 1.f;  // the V codes' scale
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int h = hh ? row1 : row0;
            if (h >= r) continue;
            const float lsum = hh ? l1 : l0;
            const size_t row = hrow + h;
            const size_t prow = prow0 + h;
            if constexpr (kFp8) {
                const float f = whole ? vsc / lsum : vsc;
#pragma unroll
                for (int sg = 0; sg < D / 16; ++sg) {
                    const float *ev = o[4 * (sg >> 1) + 2 * (sg & 1)], *od = o[4 * (sg >> 1) + 2 * (sg & 1) + 1];
                    const float v0 = ev[2 * hh] * f, v1 = od[2 * hh] * f, v2 = ev[2 * hh + 1] * f, v3 = od[2 * hh + 1] * f;
                    const int col = 16 * sg + 2 * c2;
                    if (whole)
                        *reinterpret_cast<uint2 *>(p.out + row * D + col) = make_uint2(pack_bf16x2(v0, v1), pack_bf16x2(v2, v3));
                    else
                        *reinterpret_cast<float4 *>(p.part_o + prow * D + col) = make_float4(v0, v1, v2, v3);
                }
            } else if (whole) {
                const float inv = 1.f / lsum;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    *reinterpret_cast<uint32_t *>(p.out + row * D + nt * 8 + c2) =
                        pack_bf16x2(o[nt][2 * hh] * inv, o[nt][2 * hh + 1] * inv);
            } else {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    *reinterpret_cast<float2 *>(p.part_o + prow * D + nt * 8 + c2) =
                        make_float2(o[nt][2 * hh], o[nt][2 * hh + 1]);
            }
            if (!whole && (lane & 3) == 0)
                *reinterpret_cast<float2 *>(p.part_ml + prow * 2) = make_float2(m_ref[hh] * sl2, lsum);
        }
        has = has_n;
        uc = un;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk)
#pragma unroll
            for (int e = 0; e < 4; ++e) qa[kk][e] = qn[kk][e];
    }
    if (!ok) {
        *abort = 1;
        if (lane == 0) report(p.status, PREFILL_ERR_TIMEOUT);
    }
}

// Merge of the pieces of a segment cut by CTA boundaries (the whole-page
// kernel's split work): one warp per (sequence, query head), the
// online-softmax merge rule over the pieces' (max, sum, O) -- any number of
// pieces, 32 at a time.  A segment in one piece was written by the kernel.
template <int D>
__global__ void __launch_bounds__(128) decode_merge_pieces_kernel(const DecodeParams p) {
    griddep_wait();  // the decode kernel's partials and step scan are complete
    griddep_launch_dependents();
    const int i = blockIdx.x;
    const int hq = blockIdx.y * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (hq >= p.n_head) return;
    const int ctx = p.context_lens[i];
    if (ctx < 0 || ctx > p.max_ctx || (long long)ctx + 1 > (long long)p.mbps * p.block_size) return;
    const int nslab = p.n_kv_head / TW, r = p.n_head / p.n_kv_head;
    const int g = hq / r, slab = g / TW, w = g % TW, h = hq % r;
    const int T = steps_per_cta(p.seg_cum[p.num_seqs], p.grid);
    const int ns = cdiv(ctx + 1, KS);
    const int seg_start = p.seg_cum[i] + slab * ns, seg_end = seg_start + ns;
    const int c0 = seg_start / T, np = (seg_end - 1) / T - c0 + 1;
    if (np <= 1) return;
    const size_t base_row = (size_t)(c0 + i * nslab + slab) * ((size_t)TW * r) + (size_t)w * r + h;
    const size_t pstride = (size_t)TW * r;  // rows between consecutive pieces of the segment
    constexpr int E = D / 32, PB = 4;       // the first PB pieces' O rows load with the maxima
    using V = typename std::conditional<E == 4, float4, float2>::type;
    V f[PB];
#pragma unroll
    for (int j = 0; j < PB; ++j)
        if (j < np) f[j] = __ldcg(reinterpret_cast<const V *>(p.part_o + (base_row + j * pstride) * D + lane * E));
    float2 mlane = make_float2(-CUDART_INF_F, 0.f);  // piece `lane` (first 32 pieces)
    if (lane < np) mlane = __ldcg(reinterpret_cast<const float2 *>(p.part_ml + (base_row + lane * pstride) * 2));
    float M = mlane.x;
    for (int c = lane + 32; c < np; c += 32) M = fmaxf(M, __ldcg(p.part_ml + (base_row + c * pstride) * 2));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float L = 0.f;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    auto add = [&](float wgt, const V &v) {
        const float *fv = reinterpret_cast<const float *>(&v);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(wgt, fv[e], acc[e]);
    };
    for (int cb = 0; cb < np; cb += 32) {
        float wl = 0.f;
        if (cb + lane < np) {
            const float2 ml = cb == 0 ? mlane
                                      : __ldcg(reinterpret_cast<const float2 *>(p.part_ml + (base_row + (cb + lane) * pstride) * 2));
            wl = ex2(ml.x - M);
            L += wl * ml.y;
        }
        const int nb = min(32, np - cb);
        for (int j = 0; j < nb; ++j) {
            const float wgt = __shfl_sync(0xffffffffu, wl, j);
            const int c = cb + j;
            if (c < PB) {
#pragma unroll
                for (int k = 0; k < PB; ++k)
                    if (k == c) add(wgt, f[k]);
            } else {
                add(wgt, __ldcg(reinterpret_cast<const V *>(p.part_o + (base_row + c * pstride) * D + lane * E)));
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    const float inv = 1.f / L;
    uint16_t *dst = p.out + ((size_t)i * p.n_head + hq) * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 2) *reinterpret_cast<uint32_t *>(dst + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
}

template <int D, bool kFp8>
int launch_dt(const DecodeParams &p, const CUtensorMap &tm, void *stream) {
    using L = TLay<D, kFp8>;
    const size_t smem = L::BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(paged_decode_tma_kernel<D, kFp8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return (int)e;
    const int grid = p.grid;  // steps_per_cta divides the call's steps over exactly this many CTAs
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(TTHREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = (cudaStream_t)stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, paged_decode_tma_kernel<D, kFp8>, tm, p);
    // no segment can be cut when all steps fit in one CTA's share
    const long long steps_bound = (long long)p.num_seqs * (p.n_kv_head / TW) * cdiv(p.max_ctx + 1, KS);
    if (e != cudaSuccess || steps_bound <= kMinStepsPerCta) return (int)e;
    cfg.gridDim = dim3((unsigned)p.num_seqs, (unsigned)cdiv(p.n_head, 4));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    return (int)cudaLaunchKernelEx(&cfg, decode_merge_pieces_kernel<D>, p);
}

template <int D, bool kFp8>
int launch_d(const DecodeParams &p, void *stream) {
    using L = DecLay<D, kFp8>;
    const size_t smem = L::BYTES;
    cudaError_t e =
        cudaFuncSetAttribute(paged_decode_kernel<D, kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return (int)e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long units = (long long)p.max_units * p.n_kv_head * p.num_seqs;  // a bound on the call's units
    const long long ctas_needed = (units + WARPS - 1) / WARPS;
    const long long slots = (long long)kCtasPerSm * sms;
    const int grid = (int)(ctas_needed < slots ? ctas_needed : slots);
    // programmatic dependent launches: each kernel may be scheduled while the one
    // before it on the stream drains, and waits for it before touching memory
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(DTHREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = (cudaStream_t)stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, paged_decode_kernel<D, kFp8>, p);
    if (e != cudaSuccess || p.max_units <= 1) return (int)e;
    cfg.gridDim = dim3((unsigned)p.num_seqs, (unsigned)cdiv(p.n_head, 4));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    return (int)cudaLaunchKernelEx(&cfg, decode_combine_kernel<D>, p);
}

}  // namespace

int decode_keys_per_unit(int max_ctx) {
    // units of 256 keys, longer for very long contexts (at most
    // kDecodeMaxUnits per sequence); always a multiple of the 16-key step.
    // On 64 varlen sequences 128-key units even out the keys per warp better
    // (within ~3 % of the mean against an 18 % spread), but the step measured
    // 3 % slower: half as many units means half the partials to write and
    // merge, which outweighs the spread
    int u = 256;
    while (cdiv(max_ctx + 1, u) > kDecodeMaxUnits) u *= 2;
    return u;
}

int launch_decode(const DecodeParams &p, int head_dim, bool fp8, void *stream) {
    if (fp8) return head_dim == 64 ? launch_d<64, true>(p, stream) : launch_d<128, true>(p, stream);
    return head_dim == 64 ? launch_d<64, false>(p, stream) : launch_d<128, false>(p, stream);
}

int launch_decode_tma(const DecodeParams &p, const CUtensorMap *tm, int head_dim, bool fp8, void *stream) {
    if (fp8) return launch_dt<128, true>(p, *tm, stream);
    return head_dim == 64 ? launch_dt<64, false>(p, *tm, stream) : launch_dt<128, false>(p, *tm, stream);
}

namespace {

// One warp per token: its sequence is found once (binary search over
// cu_seqlens), then the K and V rows of every kv head are quantized to e4m3
// codes (x / scale, nearest even, saturating) into the token's cache slot.
template <int D>
__global__ void __launch_bounds__(256) kv_store_fp8_kernel(const Fp8StoreParams p) {
    // launched as a programmatic dependent: the kernels before it on the stream
    // (which may still read the slots and the dense copy it writes) are complete
    griddep_wait();
    griddep_launch_dependents();
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= p.total) return;
    int lo = 0, hi = p.num_seqs - 1;  // sequence holding row t: last i with cu_seqlens[i] <= t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(&p.cu_seqlens[mid]) <= t) lo = mid; else hi = mid - 1;
    }
    const int i = lo, c0 = __ldg(&p.cu_seqlens[i]);
    if (t >= __ldg(&p.cu_seqlens[i + 1])) return;  // not a row of any sequence
    const int pos = (p.context_lens ? __ldg(&p.context_lens[i]) : 0) + (t - c0);
    const int bs = p.block_size;
    if (pos < 0 || pos / bs >= p.mbps) {
        if (lane == 0) report(p.status, PREFILL_ERR_BLOCK_TABLE);
        return;
    }
    const int page = __ldg(&p.block_table[(size_t)i * p.mbps + pos / bs]);
    if (page < 0 || page >= p.num_blocks) {
        if (lane == 0) report(p.status, PREFILL_ERR_BLOCK_TABLE);
        return;
    }
    const size_t G = p.n_kv_head;
    // the token's rows of all kv heads are contiguous (G * D elements), as are
    // its slot's codes in the K half and in the V half of the page
    constexpr int PER = 4;  // elements per lane per step
    for (int x = lane * PER; x < (int)G * D; x += 32 * PER) {
        const int g = x / D;
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            const uint16_t *src = (tt ? p.v : p.k) + (size_t)t * G * D + x;
            const float sc = __ldg(&(tt ? p.v_scale : p.k_scale)[g]);
            const uint2 v2 = __ldg(reinterpret_cast<const uint2 *>(src));
            const uint32_t c01 = quant_e4m3x2(__uint_as_float(v2.x << 16), __uint_as_float(v2.x & 0xffff0000u), sc);
            const uint32_t c23 = quant_e4m3x2(__uint_as_float(v2.y << 16), __uint_as_float(v2.y & 0xffff0000u), sc);
            uint8_t *dst = p.cache8 + (((size_t)page * 2 + tt) * bs + pos % bs) * G * D + x;
            *reinterpret_cast<uint32_t *>(dst) = c01 | (c23 << 16);
            uint8_t *dense = tt ? p.dense_v8 : p.dense_k8;
            if (dense) *reinterpret_cast<uint32_t *>(dense + (size_t)t * G * D + x) = c01 | (c23 << 16);
        }
    }
}

}  // namespace

int launch_kv_store_fp8(const Fp8StoreParams &p, int head_dim, void *stream) {
    if (p.total == 0) return 0;
    // one warp per token; a programmatic dependent launch (the kernel waits for
    // its predecessors before touching memory), so that its launch, and the
    // launch of the attention kernel that follows it, overlap the kernel before
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((p.total + 7) / 8));
    cfg.blockDim = dim3(256);
    cfg.stream = (cudaStream_t)stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    if (head_dim == 64) return (int)cudaLaunchKernelEx(&cfg, kv_store_fp8_kernel<64>, p);
    return (int)cudaLaunchKernelEx(&cfg, kv_store_fp8_kernel<128>, p);
}

}  // namespace pf
