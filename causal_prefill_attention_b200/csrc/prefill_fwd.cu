// prefill_fwd.cu -- pipelined, warp-specialised causal prefill attention for
// sm_100a, fused with the paged KV-cache write.
//
// The method is the tiled attention of hncyxsy.com/news/270449 §3.2 and §4.3:
// Q split into query blocks, K/V into kv blocks, a running row max and exp-sum
// per query row, old partial results rescaled when the max grows, P.V
// accumulated, and blocks above the causal diagonal never issued.  Only the
// final output and the KV cache reach HBM.
//
// B200 mapping (the pages target A100; this is a redesign, not their kernel):
//   * persistent grid, one CTA per SM; a work item is a pair of consecutive
//     128-row query blocks of one (sequence, head); items are ordered longest
//     first on the device from cu_seqlens and dealt to CTAs in zigzag order.
//   * warps 0-3 / 4-7: softmax for query block 0 / 1 (one TMEM lane = one
//     row per thread); they also apply the (lazy) rescale of O and store the
//     final O / l.  Warp 8: TMA producer (Q blocks, K/V ring of NST stages,
//     paged prefix gather).  Warp 9: tcgen05 MMA issuer.  Warp 10: paged KV
//     writer, a second consumer of the K/V ring that stores each item's own
//     K/V tiles from shared memory into their cache pages (TMA stores).
//     Warp 11: idle.  A call that writes an FP8 cache runs the kernel
//     without the writer (kNoWrite) and quantizes K/V in a separate pass.
//   * TMEM (512 columns): S0 | S1 | O0 | O1, 128 columns each; P (bf16) is
//     written over the first 64 columns of its S and read by the P.V MMA
//     directly from TMEM.
//   * MMA order per kv block j: PV0(j), S0(j+1), PV1(j), S1(j+1), so the
//     softmax of one query block overlaps the tensor-core work of the other.
#include <cuda_runtime.h>
#include <cstdint>
#include <map>
#include <math_constants.h>
#include <mutex>

#include "block_rule.h"
#include "params.h"
#include "sm100.cuh"
#include "../../include/prefill.h"

namespace pf {
namespace {

constexpr int BM = 128;
constexpr int BN = 128;
// K/V ring stages (each holds one K or one V tile): a template parameter of the
// kernel, 5 when the shared-memory schedule leaves room for it, else 4.
constexpr int NTHREADS = 384;
constexpr int WARP_PRODUCER = 8, WARP_MMA = 9, WARP_WRITER = 10;
constexpr uint32_t CHUNK = 128 * 128;  // 128 rows x 64 bf16, 128B-swizzled
// Threshold (log2 units) before the running max is moved and O rescaled;
// between moves P can reach 2^8, well inside fp32 / bf16 range.
constexpr float kRescaleLog2 = 8.0f;
// P (bf16 pairs) occupies the first 64 columns of its S region.
constexpr uint32_t kPOff = 0;
// Running max of a row that has seen no visible key yet (finite, far below any score).
constexpr float kNoKeyMax = -1e30f;
// Which of the 32 column pairs in each 64-column half of an unmasked block take
// their exponentials on the FMA pipe (exp2_fma2) instead of MUFU (ex2): pairs
// 0, 8, 16 and 24, one exponential in eight.  MUFU gives 16 results per clock
// per SM, as many as the tensor core needs at head_dim 128, so moving a few off
// it shortens the softmax; measured on the 8k GQA prompt: +2 to +4 % with one
// in eight, +3 % with one in four, slower beyond (the ALU pipe, at half rate,
// then limits the polynomial's clamps and exponent adds).
#ifndef PF_EXP2_EMU_MASK
#define PF_EXP2_EMU_MASK 0x01010101u
#endif
constexpr uint32_t kEmuMask = PF_EXP2_EMU_MASK;

// Shared-memory layout.  F8: the chunked mode over an FP8 cache, whose K/V tiles
// arrive as e4m3 bytes ([128 rows][D bytes], unswizzled) and are widened to
// f16 in the stage: at head_dim 128 the bytes land in the upper half of the
// stage itself (row r's bytes sit exactly where its second 64-column chunk
// goes, so each row is read before it is overwritten), at head_dim 64 in a
// separate staging area (STG, 8 KB per stage).
template <int D, int NST, bool F8 = false>
struct Lay {
    static constexpr int NCH = D / 64;
    static constexpr uint32_t TILE = NCH * CHUNK;
    static constexpr uint32_t Q0 = 0, Q1 = TILE, KV = 2 * TILE;
    static constexpr uint32_t RAW8 = 128u * D;  // e4m3 bytes of one K or V tile
    static constexpr uint32_t STG = KV + NST * TILE;
    static constexpr uint32_t BAR = STG + ((F8 && D == 64) ? NST * RAW8 : 0u);
    // barrier slots; P is handed over in two halves (columns 0..63 -> PA, 64..127 -> PB);
    // QRAW / KVRAW: the e4m3 (or bf16 Q) bytes have landed, before conversion (F8 only)
    static constexpr int B_QFULL = 0, B_QEMPTY = 2, B_KVFULL = 4, B_KVEMPTY = 4 + NST, B_SFULL = 4 + 2 * NST,
                         B_PA = 6 + 2 * NST, B_PB = 8 + 2 * NST, B_OFULL = 10 + 2 * NST, B_OEMPTY = 12 + 2 * NST,
                         B_QRAW = 14 + 2 * NST, B_KVRAW = 16 + 2 * NST, NBAR = 16 + 3 * NST;
    static constexpr uint32_t TMEM_SLOT = BAR + NBAR * 8, ABORT = TMEM_SLOT + 4;
    static constexpr uint32_t SCHED = BAR + 512;
    static_assert(ABORT + 4 <= SCHED, "barrier area overflow");
    // byte offset (from the aligned base) of the e4m3 bytes of stage st
    static constexpr uint32_t raw8(int st) { return D == 128 ? KV + st * TILE + CHUNK : STG + st * RAW8; }
};

// P to TMEM: bf16 pairs, or f16 pairs when the tensor-core operands are f16
template <bool kF16>
__device__ __forceinline__ uint32_t pack_p(float lo, float hi) {
    return kF16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
}

// P = 2^(S*scale*log2e - m*scale*log2e) for 64 columns (half h) of one row:
// packed FMA, exponentials, packed row sums into (sa*, sb*), bf16 pairs in pw.
template <int h, bool kEmu, bool kF16>
__device__ __forceinline__ void exp_half(const float (&x)[BN], float sl2, float nms, uint32_t (&pw)[32], float &sa0,
                                         float &sa1, float &sb0, float &sb1) {
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        float y0, y1, p0, p1;
        fma2(y0, y1, x[h * 64 + 2 * c], x[h * 64 + 2 * c + 1], sl2, sl2, nms, nms);
        if (kEmu && ((kEmuMask >> c) & 1u)) {
            exp2_fma2(y0, y1, p0, p1);
        } else {
            p0 = ex2(y0);
            p1 = ex2(y1);
        }
        if (c & 1) add2(sb0, sb1, p0, p1); else add2(sa0, sa1, p0, p1);
        pw[c] = pack_p<kF16>(p0, p1);
    }
}

// Row max of 128 scores: four independent chains of 3-input max.
__device__ __forceinline__ float rowmax128(const float (&x)[BN]) {
    float a0 = x[0], a1 = x[1], a2 = x[2], a3 = x[3];
#pragma unroll
    for (int c = 4; c < BN - 4; c += 8) {
        a0 = max3(a0, x[c], x[c + 1]);
        a1 = max3(a1, x[c + 2], x[c + 3]);
        a2 = max3(a2, x[c + 4], x[c + 5]);
        a3 = max3(a3, x[c + 6], x[c + 7]);
    }
    a0 = max3(a0, x[BN - 4], x[BN - 3]);
    a1 = max3(a1, x[BN - 2], x[BN - 1]);
    return fmaxf(max3(a0, a1, a2), a3);
}

// Online softmax of one kv block for one row (one thread), then P to TMEM in
// two halves, each announced on its own barrier so that the P.V MMA can start
// on the first half while the second is computed.
//
// The exponentials are taken against the running max m_run without waiting
// for this block's max: the running max only moves when the block max exceeds
// it by more than the threshold (2^8 in P), and only then is half 0 redone
// and O rescaled.  Blocks whose max stays below that bound give P up to 2^8,
// which the final O / l divides out exactly (same max for P and l).
template <int D, bool kFull, bool kF16>
__device__ __forceinline__ void softmax_block(const float (&x)[BN], bool first, float sl2, float thr, float &m_run,
                                              float &l_run, uint32_t tS, uint32_t tO, uint32_t b_pa, uint32_t b_pb,
                                              int lane) {
    float mt = first ? rowmax128(x) : 0.f;
    // a row with nothing visible in its first block (a sliding window's edge)
    // takes a finite floor as its max: its P is 0, and the first block that
    // shows it a key moves the max and rescales the empty O and l by exactly 0
    float m_ref = first ? fmaxf(mt, kNoKeyMax) : m_run;
    float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
    {
        uint32_t pw[32];
        exp_half<0, kFull, kF16>(x, sl2, -m_ref * sl2, pw, sa0, sa1, sb0, sb1);
        tmem_st32(tS + kPOff, pw);
    }
    float m_new = m_ref, alpha = first ? 0.f : 1.f;
    if (!first) {
        mt = rowmax128(x);
        const bool need = mt > m_run + thr;
        if (__any_sync(0xffffffffu, need)) {
            // the max moved by more than the threshold: redo half 0 (stored again
            // over the first attempt) and rescale O before P.V touches it
            m_new = need ? mt : m_run;
            alpha = ex2((m_run - m_new) * sl2);
            sa0 = sa1 = sb0 = sb1 = 0.f;
            {
                uint32_t pw[32];
                exp_half<0, kFull, kF16>(x, sl2, -m_new * sl2, pw, sa0, sa1, sb0, sb1);
                tmem_st32(tS + kPOff, pw);
            }
#pragma unroll 1
            for (int cc = 0; cc < D / 16; ++cc) {
                uint32_t r[16];
                tmem_ld16(tO + cc * 16, r);
#pragma unroll
                for (int c = 0; c < 16; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
                tmem_st16(tO + cc * 16, r);
            }
        }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(b_pa);
    uint32_t pw[32];
    exp_half<1, kFull, kF16>(x, sl2, -m_new * sl2, pw, sa0, sa1, sb0, sb1);
    tmem_st32(tS + kPOff + 32, pw);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(b_pb);
    l_run = l_run * alpha + ((sa0 + sa1) + (sb0 + sb1));
    m_run = m_new;
}

// Exponentials of 64 scores held in y64 (same arithmetic as exp_half),
// written to TMEM as bf16 pairs at taddr in two 16-column stores so that only
// 16 packed words are live at a time.
template <bool kEmu, bool kF16>
__device__ __forceinline__ void exp64_store(const float (&y64)[64], float sl2, float nms, uint32_t taddr,
                                            float &sa0, float &sa1, float &sb0, float &sb1) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        uint32_t pw[16];
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) {
            const int c = hh * 16 + cc;
            float y0, y1, p0, p1;
            fma2(y0, y1, y64[2 * c], y64[2 * c + 1], sl2, sl2, nms, nms);
            if (kEmu && ((kEmuMask >> c) & 1u)) {
                exp2_fma2(y0, y1, p0, p1);
            } else {
                p0 = ex2(y0);
                p1 = ex2(y1);
            }
            if (c & 1) add2(sb0, sb1, p0, p1); else add2(sa0, sa1, p0, p1);
            pw[cc] = pack_p<kF16>(p0, p1);
        }
        tmem_st16(taddr + hh * 16, pw);
    }
}

__device__ __forceinline__ float rowmax64x2(const float (&a)[64], const float (&b)[64]) {
    float a0 = a[0], a1 = a[1], a2 = b[0], a3 = b[1];
#pragma unroll
    for (int c = 2; c < 64; c += 2) {
        a0 = max3(a0, a[c], a[c + 1]);
        a2 = max3(a2, b[c], b[c + 1]);
    }
    return fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
}

// Online softmax of a block that is not the first of its range: the running
// max is already known, so the first 64 scores are exponentiated while the
// second 64 are still being read from TMEM; the block max is checked once both
// halves are in (half 0 is redone and O rescaled only if it moved past the
// threshold).  P goes to TMEM in two halves, announced on b_pa / b_pb.
template <int D, bool kFull, bool kF16>
__device__ __forceinline__ void softmax_block_stream(uint32_t tS, int lo, int lim, float sl2, float thr, float &m_run,
                                                     float &l_run, uint32_t tO, uint32_t b_pa, uint32_t b_pb,
                                                     int lane) {
    float x0[64], x1[64];
    {
        uint32_t r[64];
        tmem_ld64_nowait(tS, r);
        tmem_wait_ld_tie64(r);
#pragma unroll
        for (int c = 0; c < 64; ++c) x0[c] = __uint_as_float(r[c]);
    }
    uint32_t r1[64];
    tmem_ld64_nowait(tS + 64, r1);  // second half in flight during half 0's exponentials
    if (!kFull) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
            if (c < lo || c >= lim) x0[c] = -CUDART_INF_F;
    }
    float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
    exp64_store<kFull, kF16>(x0, sl2, -m_run * sl2, tS + kPOff, sa0, sa1, sb0, sb1);
    tmem_wait_ld_tie64(r1);
#pragma unroll
    for (int c = 0; c < 64; ++c)
        x1[c] = (kFull || (64 + c >= lo && 64 + c < lim)) ? __uint_as_float(r1[c]) : -CUDART_INF_F;
    const float mt = rowmax64x2(x0, x1);
    const bool need = mt > m_run + thr;
    float m_new = m_run, alpha = 1.f;
    if (__any_sync(0xffffffffu, need)) {
        m_new = need ? mt : m_run;
        alpha = ex2((m_run - m_new) * sl2);
        sa0 = sa1 = sb0 = sb1 = 0.f;
        exp64_store<kFull, kF16>(x0, sl2, -m_new * sl2, tS + kPOff, sa0, sa1, sb0, sb1);
#pragma unroll 1
        for (int cc = 0; cc < D / 16; ++cc) {
            uint32_t r[16];
            tmem_ld16(tO + cc * 16, r);
#pragma unroll
            for (int c = 0; c < 16; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
            tmem_st16(tO + cc * 16, r);
        }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(b_pa);
    exp64_store<kFull, kF16>(x1, sl2, -m_new * sl2, tS + kPOff + 32, sa0, sa1, sb0, sb1);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(b_pb);
    l_run = l_run * alpha + ((sa0 + sa1) + (sb0 + sb1));
    m_run = m_new;
}

// ------------------------------------------------------------------ schedule
struct Item {
    int i, h, g, qb0, c0, n, ctx;
    int nk0, nk1;  // query block 0 / 1 visits kv blocks [jf0, nk0) / [jf1, nk1)
    int two;       // second query block present
    // split of the kv range (split-KV): this item covers kv blocks [j_lo, j_hi)
    int split, nsp, j_lo, j_hi;
    int jb0, jb1;  // first kv block of query block 0 / 1 inside this split (j_lo without a window)
    bool skip;     // a split index beyond this pair's useful split count: no work
    __device__ __forceinline__ int nk(int s) const { return s ? nk1 : nk0; }
    __device__ __forceinline__ int nmax() const { return nk0 > nk1 ? nk0 : nk1; }
    // first / end of query block s's blocks inside this split
    __device__ __forceinline__ int beg(int s) const { return s ? jb1 : jb0; }
    __device__ __forceinline__ int end(int s) const { return nk(s) < j_hi ? nk(s) : j_hi; }
};

// Useful number of splits of a pair whose kv range has nmax blocks: at most
// nsplit, and every split keeps at least kMinSplitBlocks blocks (so query block
// 0, which ends one block before query block 1, and query block 1, which
// starts at most two blocks after query block 0 under a sliding window, always
// have work in every split).
constexpr int kMinSplitBlocks = 4;
__host__ __device__ __forceinline__ int useful_splits(int nmax, int nsplit) {
    const int m = nmax / kMinSplitBlocks;
    return nsplit < m ? nsplit : (m > 1 ? m : 1);
}

__device__ __forceinline__ int seq_pairs(const FwdParams &p, int i, bool *bad) {
    const int c0 = p.cu_seqlens[i], c1 = p.cu_seqlens[i + 1];
    const int n = c1 - c0;
    const int ctx = p.context_lens ? p.context_lens[i] : 0;
    const bool bl = n < 0 || n > p.max_q || c0 < 0 || c1 > p.total;
    const bool bc = ctx < 0 || (long long)ctx + n > (long long)p.mbps * p.block_size;
    if (bl || bc) {
        *bad = true;
        return 0;
    }
    return cdiv(n, 2 * BM);
}

// Work items are ordered sequence-major: sequences by pair count, descending
// (ties by index), then the pair index p descending, then the head.  Longest
// causal rows come first (a longest-processing-time order for the persistent
// grid) and the items of one sequence run close together in time, so its K/V
// stays in L2 while its heads and pairs reuse it.
//   cnt[c]   sequences with exactly c pairs            (c = 1 .. P)
//   start[c] sequences with more than c pairs          (= first sorted slot of bucket c)
//   B[c]     items of sequences with more than c pairs (= first item of bucket c)
//   perm     sequence indices sorted by pair count, descending, stable
// The kernel is compiled per mode: kWin runs a sliding window (p.window
// keys), kChunk reads a cached prefix (p.context_lens).  Without them every
// window term, and every prefix branch (the context is the constant 0), folds
// away at compile time.  kNoWrite leaves the cache alone (no writer warp; the
// K/V ring is released by the MMA warp alone).  kFp8 (with kChunk, kNoWrite)
// reads every key and value as e4m3 codes -- the prefix from the FP8 cache's
// pages, the chunk's own rows from a dense copy of their codes -- widened to
// f16 in shared memory by warps 10-11, with Q converted to f16 the same way,
// so the tensor cores run kind::f16 on f16 operands (P is packed as f16 too).
constexpr int kModeWindow = 1, kModeChunk = 2, kModeNoWrite = 4, kModeFp8 = 8;
template <bool kWin, bool kChunk>
__device__ __forceinline__ Item decode_item(const FwdParams &p, const int *B, const int *start, const uint16_t *perm,
                                            int P, int u_split) {
    const int u = u_split / p.nsplit;
    const int split = u_split - u * p.nsplit;
    int lo = 1, hi = P;  // smallest c in [1, P] with B[c] <= u
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (B[mid] <= u) hi = mid; else lo = mid + 1;
    }
    const int c = lo;
    const int v = u - B[c];
    const int per_seq = p.n_head * c;
    const int ks = v / per_seq;
    const int w = v - ks * per_seq;
    const int pw = w / p.n_head;
    Item it;
    it.h = w - pw * p.n_head;
    it.i = perm[start[c] + ks];
    it.g = it.h / p.group;
    it.qb0 = 2 * (c - 1 - pw);
    it.c0 = p.cu_seqlens[it.i];
    it.n = p.cu_seqlens[it.i + 1] - it.c0;
    it.ctx = kChunk ? p.context_lens[it.i] : 0;
    it.two = (it.qb0 + 1) * BM < it.n;
    it.nk0 = num_kv_blocks(it.qb0, it.ctx, it.n, BM, BN);
    it.nk1 = it.two ? num_kv_blocks(it.qb0 + 1, it.ctx, it.n, BM, BN) : 0;
    const int nmax = it.nmax();
    it.split = split;
    if (!kWin) {
        it.nsp = useful_splits(nmax, p.nsplit);
        it.skip = split >= it.nsp;
        it.j_lo = (split * nmax) / it.nsp;
        it.j_hi = ((split + 1) * nmax) / it.nsp;
        it.jb0 = it.jb1 = it.j_lo;
    } else {
        const int jf0 = first_kv_block(it.qb0, it.ctx, it.n, BM, BN, p.window);
        const int jf1 = it.two ? first_kv_block(it.qb0 + 1, it.ctx, it.n, BM, BN, p.window) : jf0;
        const int nrange = nmax - jf0;  // the pair's kv range [jf0, nmax)
        it.nsp = useful_splits(nrange, p.nsplit);
        it.skip = split >= it.nsp;
        it.j_lo = jf0 + (split * nrange) / it.nsp;
        it.j_hi = jf0 + ((split + 1) * nrange) / it.nsp;
        it.jb0 = it.j_lo;  // jf0 <= j_lo
        it.jb1 = jf1 > it.j_lo ? jf1 : it.j_lo;
    }
    return it;
}

__device__ __forceinline__ int zigzag(int k, int c, int G) { return k * G + ((k & 1) ? (G - 1 - c) : c); }

// ------------------------------------------------------------------ waits
// Bounded wait that also stops when another role has given up; the first
// role to run out of time raises the CTA's abort flag.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort) {
    if (mbar_wait(bar, parity, abort)) return true;
    *abort = 1;
    return false;
}

// Register split (the launch gives 384 threads x 168 = 64,512 registers):
// softmax warpgroups 2 x 128 x 208 + control warpgroup 128 x 88 = 64,512.
__device__ __forceinline__ void setmaxnreg_softmax() { asm volatile("setmaxnreg.inc.sync.aligned.u32 208;"); }
__device__ __forceinline__ void setmaxnreg_control() { asm volatile("setmaxnreg.dec.sync.aligned.u32 88;"); }

// ------------------------------------------------------------------ kernel
template <int D, int NST, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
prefill_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_cache,
                   const FwdParams p, const int P) {
    constexpr bool kWin = (MODE & kModeWindow) != 0, kChunk = (MODE & kModeChunk) != 0;
    constexpr bool kWrite = (MODE & kModeNoWrite) == 0;
    constexpr bool kFp8 = (MODE & kModeFp8) != 0;
    using L = Lay<D, NST, kFp8>;
    // a bf16 chunk appends to the cache it reads its prefix from; an FP8 chunk's
    // codes are stored before the kernel runs
    static_assert(kWrite || !kChunk || kFp8, "a chunk's prefix is read from the cache that it appends to");
    static_assert(!kFp8 || (kChunk && !kWrite && !kWin), "the FP8 mode is the chunked mode without a window");
    constexpr uint32_t IDESC_QK = kFp8 ? idesc_f16_f32(BM, BN, false, false) : idesc_bf16_f32(BM, BN, false, false);
    constexpr uint32_t IDESC_PV = kFp8 ? idesc_f16_f32(BM, D, false, true) : idesc_bf16_f32(BM, D, false, true);

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    volatile int *abort = reinterpret_cast<volatile int *>(gbase + L::ABORT);
    int *B = reinterpret_cast<int *>(gbase + L::SCHED);  // [P + 1]
    int *start = B + (P + 1);                            // [P + 1]
    int *cur = start + (P + 1);                          // [P + 1]
    uint16_t *perm = reinterpret_cast<uint16_t *>(cur + (P + 1));
    auto bar = [&](int idx) -> uint32_t { return base + L::BAR + 8u * idx; };

    // ---------------- set-up: barriers, TMEM, schedule
    if (tid == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        if (kWrite || kChunk) tma_prefetch_desc(&tm_cache);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(L::B_QFULL + s), kFp8 ? 2 : 1);  // TMA (or the two converter warps)
            if (kFp8) mbar_init(bar(L::B_QRAW + s), 1);
            mbar_init(bar(L::B_QEMPTY + s), 1);
            mbar_init(bar(L::B_SFULL + s), 1);
            mbar_init(bar(L::B_PA + s), 4);
            mbar_init(bar(L::B_PB + s), 4);
            mbar_init(bar(L::B_OFULL + s), 1);
            mbar_init(bar(L::B_OEMPTY + s), 4);
        }
        for (int s = 0; s < NST; ++s) {
            mbar_init(bar(L::B_KVFULL + s), kFp8 ? 2 : 1);
            if (kFp8) mbar_init(bar(L::B_KVRAW + s), 1);
            mbar_init(bar(L::B_KVEMPTY + s), kWrite ? 2 : 1);  // MMA commit (+ KV writer)
        }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(base + L::TMEM_SLOT, 512);
        tmem_relinquish();
    }
    for (int x = tid; x <= P; x += NTHREADS) cur[x] = 0;
    __syncthreads();
    // Nothing above read global memory.  From here on the previous kernels on
    // the stream (e.g. the chunk before this one, whose K/V this call reads from
    // the cache) are complete and their writes visible; the next launch may be
    // scheduled now and waits the same way for this one.
    griddep_wait();
    griddep_launch_dependents();
    {
        bool bad = false;
        for (int i = tid; i < p.num_seqs; i += NTHREADS) {
            const int c = seq_pairs(p, i, &bad);
            if (c > 0) atomicAdd(&cur[c], 1);
        }
        if (bad && blockIdx.x == 0) report(p.status, PREFILL_ERR_SHAPE);
    }
    __syncthreads();
    if (warp == 0) {
        // Suffix scans over c = P .. 0 (lane 0 holds the largest c of a chunk):
        //   start[c] = sum_{c' > c} cnt[c'],  B[c] = n_head * sum_{c' > c} c' cnt[c'].
        int carry_s = 0, carry_b = 0;
        for (int top = P; top >= 0; top -= 32) {
            const int c = top - lane;
            const int hc = c >= 0 ? cur[c] : 0;
            int incl = hc, inclw = hc * (c >= 0 ? c : 0);
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, off);
                const int tw = __shfl_up_sync(0xffffffffu, inclw, off);
                if (lane >= off) {
                    incl += t;
                    inclw += tw;
                }
            }
            if (c >= 0) {
                start[c] = carry_s + incl - hc;
                cur[c] = carry_s + incl - hc;
                B[c] = (carry_b + inclw - hc * c) * p.n_head;
            }
            carry_s += __shfl_sync(0xffffffffu, incl, 31);
            carry_b += __shfl_sync(0xffffffffu, inclw, 31);
        }
        __syncwarp();
        // stable counting sort of sequences by pair count, descending
        for (int b0 = 0; b0 < p.num_seqs; b0 += 32) {
            const int i = b0 + lane;
            bool bad = false;
            const int c = i < p.num_seqs ? seq_pairs(p, i, &bad) : 0;
            const unsigned act = __ballot_sync(0xffffffffu, c > 0);
            if (c > 0) {
                const unsigned grp = __match_any_sync(act, c);
                const int rank = __popc(grp & ((1u << lane) - 1u));
                perm[cur[c] + rank] = (uint16_t)i;
                __syncwarp(grp);
                if (rank == 0) cur[c] += __popc(grp);
            }
            __syncwarp();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int total = B[0] * p.nsplit;
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(gbase + L::TMEM_SLOT);
    const int G = gridDim.x, cta = blockIdx.x;

    if (warp < 8) {
        // ================= softmax / rescale / epilogue for query block s
        setmaxnreg_softmax();
        const int s = warp >> 2;
        const int row = tid & 127;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + 128u * s + lane_off;
        const uint32_t tO = tmem + 256u + 128u * s + lane_off;
        const uint32_t b_sfull = bar(L::B_SFULL + s), b_pa = bar(L::B_PA + s), b_pb = bar(L::B_PB + s);
        const uint32_t b_ofull = bar(L::B_OFULL + s), b_oempty = bar(L::B_OEMPTY + s);
        uint32_t ph_s = 0, ph_o = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int u = zigzag(k, cta, G);
            if (u >= total) break;
            const Item it = decode_item<kWin, kChunk>(p, B, start, perm, P, u);
            if (it.skip || (s == 1 && !it.two)) continue;
            const int qb = it.qb0 + s;
            // scores in log2 units: scale * log2(e), times the kv head's key factor when one is folded in
            const float sl2 = p.k_fold ? p.scale_log2 * __ldg(&p.k_fold[it.g]) : p.scale_log2;
            const float thr = kRescaleLog2 / sl2;  // the threshold in raw score units
            const float vf = p.v_fold ? __ldg(&p.v_fold[it.g]) : 1.f;
            const int jb = kWin ? it.beg(s) : it.j_lo, je = it.end(s);
            float m_run = -CUDART_INF_F, l_run = 0.f;
            for (int j = jb; j < je; ++j) {
                if (!wait_bar(b_sfull, ph_s, abort)) { ok = false; break; }
                ph_s ^= 1;
                tc_fence_after();
                const KvBlock kb = kv_block(qb, j, it.ctx, it.n, BM, BN, kWin ? p.window : 0);
                const int lim = kb.full ? BN : col_limit(kb, row, BN);
                const int lo = (kWin && !kb.full) ? col_lo(kb, row, BN) : 0;
                if (j != jb) {
                    if (kb.full)
                        softmax_block_stream<D, true, kFp8>(tS, lo, lim, sl2, thr, m_run, l_run, tO, b_pa, b_pb, lane);
                    else
                        softmax_block_stream<D, false, kFp8>(tS, lo, lim, sl2, thr, m_run, l_run, tO, b_pa, b_pb,
                                                             lane);
                } else {
                    float x[BN];
                    {
                        uint32_t r[BN];
                        tmem_ld128(tS, r);
#pragma unroll
                        for (int c = 0; c < BN; ++c)
                            x[c] = (c >= lo && c < lim) ? __uint_as_float(r[c]) : -CUDART_INF_F;
                    }
                    if (kb.full)
                        softmax_block<D, true, kFp8>(x, true, sl2, thr, m_run, l_run, tS, tO, b_pa, b_pb, lane);
                    else
                        softmax_block<D, false, kFp8>(x, true, sl2, thr, m_run, l_run, tS, tO, b_pa, b_pb, lane);
                }
            }
            if (!ok) break;
            // final O / l -> bf16 rows of out
            if (!wait_bar(b_ofull, ph_o, abort)) { ok = false; break; }
            ph_o ^= 1;
            tc_fence_after();
            const int a = qb * BM + row;
            if (p.part_nsp && it.h == 0 && it.split == 0 && a < it.n)
                p.part_nsp[it.c0 + a] = (p.epoch << 4) | (uint32_t)it.nsp;
            if (it.nsp > 1) {
                // split-KV: unnormalised O, the running max (log2 units) and the
                // exp-sum go to the workspace; the combine kernel merges the splits.
                // O chunk-major ([split][head][column / 4][row]): a warp's 32 rows
                // of one 4-column chunk are 512 contiguous bytes
                const size_t sh = (size_t)it.split * p.n_head + it.h;
                float4 *po = reinterpret_cast<float4 *>(p.part_o) + sh * (D / 4) * p.total + (it.c0 + a);
                uint32_t r[32];
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    tmem_ld32(tO + cc * 32, r);
                    if (p.v_fold) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * vf);
                    }
                    if (a < it.n) {
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            po[(size_t)(cc * 8 + c) * p.total] = make_float4(
                                __uint_as_float(r[4 * c]), __uint_as_float(r[4 * c + 1]), __uint_as_float(r[4 * c + 2]),
                                __uint_as_float(r[4 * c + 3]));
                    }
                }
                if (a < it.n)
                    *reinterpret_cast<float2 *>(p.part_ml + (sh * p.total + it.c0 + a) * 2) = make_float2(m_run * sl2, l_run);
            } else {
            const float inv_l = vf / l_run;
            uint16_t *dst = p.out + ((size_t)(it.c0 + a) * p.n_head + it.h) * D;
            {
                uint32_t r[32];
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    tmem_ld32(tO + cc * 32, r);
                    uint32_t w[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        w[c] = pack_bf16x2(__uint_as_float(r[2 * c]) * inv_l, __uint_as_float(r[2 * c + 1]) * inv_l);
                    if (a < it.n) {
                        uint4 *d4 = reinterpret_cast<uint4 *>(dst + cc * 32);
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            d4[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                    }
                }
            }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b_oempty);
        }
        if (!ok && (tid & 127) == 0) report(p.status, PREFILL_ERR_TIMEOUT);
    } else {
        setmaxnreg_control();
        if (warp == WARP_PRODUCER) {
            // ================= TMA producer (all lanes loop; lane 0 issues)
            const int bs = p.block_size;
            int stage = 0;
            uint32_t phase = 0, ph_qe = 0;  // bit s: phase of Q block s
            // stages / Q buffers filled at least once, and the phase of their last
            // fill: drained before exit so that no copy is in flight when the CTA ends
            uint32_t kv_filled = 0, kv_lastph = 0, q_filled = 0, q_lastph = 0;
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int u = zigzag(k, cta, G);
                if (u >= total) break;
                const Item it = decode_item<kWin, kChunk>(p, B, start, perm, P, u);
                if (it.skip) continue;
                const int ns = it.two ? 2 : 1;
                for (int s = 0; s < ns; ++s) {
                    if (!wait_bar(bar(L::B_QEMPTY + s), ((ph_qe >> s) & 1u) ^ 1u, abort)) { ok = false; break; }
                    if (p.test_stall && cta == 0 && k == 0 && s == 0) {
                        // test hook: withhold this Q tile so that the MMA warp's wait expires
                        ph_qe ^= 1u << s;
                        continue;
                    }
                    q_filled |= 1u << s;
                    q_lastph = (q_lastph & ~(1u << s)) | (((ph_qe >> s) & 1u) << s);
                    ph_qe ^= 1u << s;
                    if (lane == 0) {
                        const uint32_t b = bar(kFp8 ? L::B_QRAW + s : L::B_QFULL + s);
                        mbar_expect_tx(b, L::TILE);
                        tma_load_4d(base + (s ? L::Q1 : L::Q0), &tm_q, b, 0, it.h, it.c0 + (it.qb0 + s) * BM, 0);
                    }
                }
                // Prefix blocks: lane x < (whole pages) * NCH issues the box of page
                // x / NCH, chunk x % NCH (bs >= 16, so at most 16 boxes per block).
                // Its page number is read one block ahead, so that the block-table
                // load overlaps the previous block's copies, and serves both K and V.
                auto lane_page = [&](int jj) -> int {
                    const KvBlock kk = kv_block(it.qb0, jj, it.ctx, it.n, BM, BN, 0);
                    if (kFp8) {
                        if (!kk.prefix || lane >= cdiv(kk.lim_const, bs)) return 0;
                        return __ldg(&p.block_table[(size_t)it.i * p.mbps + kk.key_begin / bs + lane]);
                    }
                    if (!kk.prefix || lane >= (kk.lim_const / bs) * L::NCH) return 0;
                    return __ldg(&p.block_table[(size_t)it.i * p.mbps + kk.key_begin / bs + lane / L::NCH]);
                };
                const int np = cdiv(it.ctx, BN);  // prefix blocks come first
                int page_next = it.j_lo < np ? lane_page(it.j_lo) : 0;
                for (int j = it.j_lo; j < it.j_hi && ok; ++j) {
                    const KvBlock kb = kv_block(it.qb0, j, it.ctx, it.n, BM, BN, 0);  // key range only
                    int page_cur = page_next;
                    if (j + 1 < it.j_hi && j + 1 < np) page_next = lane_page(j + 1);
                    if (page_cur < 0 || page_cur >= p.num_blocks) {
                        report(p.status, PREFILL_ERR_BLOCK_TABLE);
                        page_cur = p.num_blocks;  // outside the map: the box reads zeros
                    }
                    for (int t = 0; t < 2; ++t) {  // t = 0: K, t = 1: V
                        if (!wait_bar(bar(L::B_KVEMPTY + stage), phase ^ 1, abort)) { ok = false; break; }
                        const uint32_t dst = base + L::KV + stage * L::TILE;
                        const uint32_t b = bar(L::B_KVFULL + stage);
                        kv_filled |= 1u << stage;
                        kv_lastph = (kv_lastph & ~(1u << stage)) | (phase << stage);
                        if (kFp8) {
                            // e4m3 bytes into the stage's staging bytes; the converter warps
                            // widen them (rows past the valid keys are zeroed there)
                            const uint32_t d8 = base + L::raw8(stage);
                            const uint32_t b8 = bar(L::B_KVRAW + stage);
                            if (!kb.prefix) {
                                if (lane == 0) {
                                    mbar_expect_tx(b8, L::RAW8);
                                    tma_load_4d(d8, t ? &tm_v : &tm_k, b8, 0, it.g, it.c0 + kb.src_row, 0);
                                }
                            } else {
                                // whole pages, one box per lane (the last page may be partly valid)
                                const int pages = cdiv(kb.lim_const, bs);
                                if (lane == 0) mbar_expect_tx(b8, (uint32_t)(pages * bs * D));
                                __syncwarp();
                                if (lane < pages)
                                    tma_load_4d(d8 + lane * bs * D, &tm_cache, b8, 0, it.g, 0, page_cur * 2 + t);
                            }
                        } else if (!kb.prefix) {
                            if (lane == 0) {
                                mbar_expect_tx(b, L::TILE);
                                tma_load_4d(dst, t ? &tm_v : &tm_k, b, 0, it.g, it.c0 + kb.src_row, 0);
                            }
                        } else {
                            // prefix: whole pages by TMA; the rest of the block (a partly
                            // valid page, rows past the prefix) by plain loads and zeros
                            const int npos = kb.lim_const;
                            const int full_pages = npos / bs;
                            const int r0 = full_pages * bs;
                            if (r0 < BN) {
                                const int units = (BN - r0) * 8 * L::NCH;
                                for (int x = lane; x < units; x += 32) {
                                    const int rr = r0 + x / (8 * L::NCH);
                                    const int ch = (x / 8) % L::NCH;
                                    const int un = x % 8;
                                    uint4 val = make_uint4(0, 0, 0, 0);
                                    if (rr < npos) {
                                        const int P_ = kb.key_begin + rr;
                                        const int page = p.block_table[(size_t)it.i * p.mbps + P_ / bs];
                                        if (page >= 0 && page < p.num_blocks) {
                                            const size_t off =
                                                ((((size_t)page * 2 + t) * bs + P_ % bs) * p.n_kv_head + it.g) * D +
                                                ch * 64 + un * 8;
                                            val = *reinterpret_cast<const uint4 *>(p.cache + off);
                                        } else {
                                            report(p.status, PREFILL_ERR_BLOCK_TABLE);
                                        }
                                    }
                                    uint8_t *d = gbase + (dst - base) + ch * CHUNK + rr * 128 + ((un ^ (rr & 7)) << 4);
                                    *reinterpret_cast<uint4 *>(d) = val;
                                }
                                fence_proxy_async_smem();
                                __syncwarp();
                            }
                            // one (page, 64-column chunk) box per lane: a single thread pays
                            // ~300 clocks per TMA issue, lanes issuing together overlap it
                            if (lane == 0) mbar_expect_tx(b, (uint32_t)(full_pages * bs * 128 * L::NCH));
                            __syncwarp();
                            if (lane < full_pages * L::NCH) {
                                const int pg = lane / L::NCH, ch = lane % L::NCH;
                                tma_load_4d(dst + ch * CHUNK + pg * bs * 128, &tm_cache, b, ch * 64, it.g, 0,
                                            page_cur * 2 + t);
                            }
                        }
                        if (++stage == NST) { stage = 0; phase ^= 1; }
                    }
                }
            }
            // drain: every copy this warp issued has landed before the CTA can exit
            // (immediate on the normal path, where the consumers waited for them)
            for (int st = 0; st < NST; ++st)
                if ((kv_filled >> st) & 1u)
                    mbar_wait(bar(kFp8 ? L::B_KVRAW + st : L::B_KVFULL + st), (kv_lastph >> st) & 1u);
            for (int s = 0; s < 2; ++s)
                if ((q_filled >> s) & 1u)
                    mbar_wait(bar(kFp8 ? L::B_QRAW + s : L::B_QFULL + s), (q_lastph >> s) & 1u);
            if (!ok && lane == 0) report(p.status, PREFILL_ERR_TIMEOUT);
        } else if (warp == WARP_MMA) {
            // ================= tcgen05 MMA issuer: the whole warp runs the loop with
            // warp-uniform descriptors; one elected lane issues each instruction.
            int stage = 0;
            // per-query-block phase bits (bit s) and "O already used" bits
            uint32_t phase = 0, ph_qf = 0, ph_pf = 0, ph_oe = 0, used = 0;
            bool ok = true;
            auto wait_all = [&](uint32_t b, uint32_t par) {
                return __all_sync(0xffffffffu, wait_bar(b, par, abort));
            };
            const uint64_t dq0 = smem_desc_sw128(base + L::Q0, 16, 1024);
            const uint64_t dq1 = smem_desc_sw128(base + L::Q1, 16, 1024);
            auto issue_s = [&](int s, int kst) {
                const uint64_t dq = s ? dq1 : dq0;
                const uint64_t dk = smem_desc_sw128(base + L::KV + kst * L::TILE, 16, 1024);
                const uint32_t d = tmem + 128u * s;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = (uint64_t)(((kk >> 2) * CHUNK + (kk & 3) * 32) >> 4);
                    mma_ss_elect(d, dq + off, dk + off, IDESC_QK, kk > 0);
                }
            };
            // k-steps [k0, k0 + 4) of O_s += P_s V (16 keys each): one half of P
            auto issue_pv = [&](int s, int vst, bool acc, int k0) {
                const uint64_t dv = smem_desc_sw128(base + L::KV + vst * L::TILE, CHUNK, 1024);
                const uint32_t d = tmem + 256u + 128u * s, a = tmem + 128u * s;
#pragma unroll
                for (int kk = k0; kk < k0 + BN / 32; ++kk)
                    mma_ts_elect(d, a + kk * 8, dv + (uint64_t)((kk * 2048) >> 4), IDESC_PV, (acc || kk > 0) ? 1u : 0u);
            };
            for (int k = 0; ok; ++k) {
                const int u = zigzag(k, cta, G);
                if (u >= total) break;
                const Item it = decode_item<kWin, kChunk>(p, B, start, perm, P, u);
                if (it.skip) continue;
                const int ns = it.two ? 2 : 1;
                const int j0 = it.j_lo, jend = it.j_hi;
                for (int s = 0; s < ns && ok; ++s) {
                    ok = wait_all(bar(L::B_QFULL + s), (ph_qf >> s) & 1u);
                    ph_qf ^= 1u << s;
                }
                if (!ok) break;
                // K_0
                const int kst = stage;
                const uint32_t kph = phase;
                if (++stage == NST) { stage = 0; phase ^= 1; }
                if (!wait_all(bar(L::B_KVFULL + kst), kph)) { ok = false; break; }
                tc_fence_after();
                for (int s = 0; s < ns; ++s) {
                    if (kWin && it.beg(s) != j0) continue;  // a windowed query block 1 may start later
                    issue_s(s, kst);
                    tc_commit_elect(bar(L::B_SFULL + s));
                }
                tc_commit_elect(bar(L::B_KVEMPTY + kst));
                for (int j = j0; j < jend && ok; ++j) {
                    const int vst = stage;
                    const uint32_t vph = phase;
                    if (++stage == NST) { stage = 0; phase ^= 1; }
                    int nst = -1;
                    uint32_t nph = 0;
                    if (j + 1 < jend) {
                        nst = stage;
                        nph = phase;
                        if (++stage == NST) { stage = 0; phase ^= 1; }
                    }
                    if (!wait_all(bar(L::B_KVFULL + vst), vph)) { ok = false; break; }
                    bool next_ready = false;
                    for (int s = 0; s < ns; ++s) {
                        // query block s visits [jb, je) of this split
                        const int jb = kWin ? it.beg(s) : j0, je = it.end(s);
                        const bool pv = (!kWin || j >= jb) && j < je;
                        if (pv) {
                            if (!wait_all(bar(L::B_PA + s), (ph_pf >> s) & 1u)) { ok = false; break; }
                            if (j == jb && ((used >> s) & 1u)) {
                                if (!wait_all(bar(L::B_OEMPTY + s), (ph_oe >> s) & 1u)) { ok = false; break; }
                                ph_oe ^= 1u << s;
                            }
                            tc_fence_after();
                            issue_pv(s, vst, j > jb, 0);
                            if (!wait_all(bar(L::B_PB + s), (ph_pf >> s) & 1u)) { ok = false; break; }
                            ph_pf ^= 1u << s;
                            tc_fence_after();
                            issue_pv(s, vst, j > jb, BN / 32);
                        }
                        if ((!kWin || j + 1 >= jb) && j + 1 < je) {
                            if (!next_ready) {
                                if (!wait_all(bar(L::B_KVFULL + nst), nph)) { ok = false; break; }
                                tc_fence_after();
                                next_ready = true;
                            }
                            issue_s(s, nst);
                            tc_commit_elect(bar(L::B_SFULL + s));
                        } else if (pv) {
                            tc_commit_elect(bar(L::B_OFULL + s));
                            tc_commit_elect(bar(L::B_QEMPTY + s));
                        }
                    }
                    if (!ok) break;
                    tc_commit_elect(bar(L::B_KVEMPTY + vst));
                    if (nst >= 0) {
                        if (!next_ready) {  // no query block needed K_{j+1}: still consume the stage in order
                            if (!wait_all(bar(L::B_KVFULL + nst), nph)) { ok = false; break; }
                        }
                        tc_commit_elect(bar(L::B_KVEMPTY + nst));
                    }
                }
                used |= it.two ? 3u : 1u;
            }
            if (!ok && lane == 0) report(p.status, PREFILL_ERR_TIMEOUT);
            __syncwarp();
        } else if (kFp8 && warp >= WARP_WRITER) {
            // ================= converters (FP8 mode, warps 10-11): each Q tile bf16 -> f16
            // in place, each K/V tile e4m3 -> f16 into the stage; every e4m3 value is
            // exact in f16, and rows past the block's valid keys become zeros (their
            // bytes may be another sequence's, a stale page's, or anything)
            const int cw = warp - WARP_WRITER;  // 0 or 1
            int stage = 0;
            uint32_t phase = 0, ph_qr = 0;
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int u = zigzag(k, cta, G);
                if (u >= total) break;
                const Item it = decode_item<kWin, kChunk>(p, B, start, perm, P, u);
                if (it.skip) continue;
                const int ns = it.two ? 2 : 1;
                for (int s = 0; s < ns; ++s) {
                    if (!wait_bar(bar(L::B_QRAW + s), (ph_qr >> s) & 1u, abort)) { ok = false; break; }
                    ph_qr ^= 1u << s;
                    uint4 *q4 = reinterpret_cast<uint4 *>(gbase + (s ? L::Q1 : L::Q0));
                    for (int x = cw * 32 + lane; x < (int)(L::TILE / 16); x += 64) {
                        uint4 w = q4[x];
                        uint32_t *wv = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            wv[e] = pack_f16x2(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xffff0000u));
                        q4[x] = w;
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(L::B_QFULL + s));
                }
                if (!ok) break;
                for (int j = it.j_lo; j < it.j_hi && ok; ++j) {
                    const KvBlock kb = kv_block(it.qb0, j, it.ctx, it.n, BM, BN, 0);
                    const int valid = kb.prefix ? kb.lim_const : imin(BN, it.n - kb.src_row);
                    for (int t = 0; t < 2; ++t) {
                        if (!wait_bar(bar(L::B_KVRAW + stage), phase, abort)) { ok = false; break; }
                        const uint8_t *src8 = gbase + L::raw8(stage);
                        uint8_t *tile = gbase + L::KV + stage * L::TILE;
                        // D = 128: 8 lanes per 128-byte row, 4 rows per warp per round
                        // D = 64: 4 lanes per 64-byte row, 8 rows per warp per round
                        // Four rounds at a time: their loads are issued together, then
                        // (after every lane's loads) their rows are written.  A row's
                        // second chunk overlaps only that row's own bytes (D = 128).
                        constexpr int LPR = D / 16, RPW = 32 / LPR, ROUNDS = BN / (2 * RPW), BATCH = 4;
                        const int qp = lane % LPR;  // columns 16 qp .. 16 qp + 15
                        const int ch = qp >> 2, u0 = (qp & 3) * 2;
#pragma unroll 1
                        for (int rb = 0; rb < ROUNDS; rb += BATCH) {
                            uint4 c[BATCH];
#pragma unroll
                            for (int b = 0; b < BATCH; ++b) {
                                const int r = (rb + b) * 2 * RPW + cw * RPW + lane / LPR;
                                c[b] = r < valid ? *reinterpret_cast<const uint4 *>(src8 + r * D + qp * 16)
                                                 : make_uint4(0, 0, 0, 0);
                            }
                            __syncwarp();  // the rows' bytes are read before their second chunks are written
#pragma unroll
                            for (int b = 0; b < BATCH; ++b) {
                                const int r = (rb + b) * 2 * RPW + cw * RPW + lane / LPR;
                                uint32_t h[8];
                                e4m3x4_to_f16x2x2_exact(c[b].x, h[0], h[1]);
                                e4m3x4_to_f16x2x2_exact(c[b].y, h[2], h[3]);
                                e4m3x4_to_f16x2x2_exact(c[b].z, h[4], h[5]);
                                e4m3x4_to_f16x2x2_exact(c[b].w, h[6], h[7]);
                                uint8_t *row = tile + ch * CHUNK + r * 128;
                                *reinterpret_cast<uint4 *>(row + ((u0 ^ (r & 7)) << 4)) =
                                    make_uint4(h[0], h[1], h[2], h[3]);
                                *reinterpret_cast<uint4 *>(row + (((u0 + 1) ^ (r & 7)) << 4)) =
                                    make_uint4(h[4], h[5], h[6], h[7]);
                            }
                            __syncwarp();
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(L::B_KVFULL + stage));
                        if (++stage == NST) { stage = 0; phase ^= 1; }
                    }
                }
            }
            if (!ok && lane == 0) report(p.status, PREFILL_ERR_TIMEOUT);
            __syncwarp();
        } else if (kWrite && warp == WARP_WRITER) {
            // ================= paged KV write, fused with the K/V staging: the writer
            // consumes every stage of the ring; the item's own (diagonal) K and V
            // tiles are stored from shared memory straight into their cache pages,
            // whole pages by TMA, a ragged last page (or pages not aligned to the
            // tile) by plain stores.  One query head per kv group writes.
            const int bs = p.block_size;
            const size_t G_ = p.n_kv_head;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int u = zigzag(k, cta, G);
                if (u >= total) break;
                const Item it = decode_item<kWin, kChunk>(p, B, start, perm, P, u);
                if (it.skip) continue;
                const int np = cdiv(it.ctx, BN);
                const bool writes = (it.h % p.group) == 0;
                for (int j = it.j_lo; j < it.j_hi && ok; ++j) {
                    const int jc = j - np;  // chunk block index (negative: prefix)
                    const bool own = writes && (jc == it.qb0 || (it.two && jc == it.qb0 + 1));
                    for (int t = 0; t < 2; ++t) {
                        if (!wait_bar(bar(L::B_KVFULL + stage), phase, abort)) { ok = false; break; }
                        if (own) {
                            const uint32_t src = base + L::KV + stage * L::TILE;
                            const int a0 = jc * BN;                      // first chunk row of the tile
                            const int rows = min(BN, it.n - a0);         // valid rows
                            const int P0 = it.ctx + a0;                  // absolute position of row 0
                            const bool aligned = (P0 % bs) == 0;
                            const int tma_rows = aligned ? (rows / bs) * bs : 0;
                            // one (page, chunk) store per lane, issued together
                            const int nst = (tma_rows / bs) * L::NCH;
                            for (int x = lane; x < nst; x += 32) {
                                const int r = (x / L::NCH) * bs, ch = x % L::NCH;
                                const int page = p.block_table[(size_t)it.i * p.mbps + (P0 + r) / bs];
                                if (page < 0 || page >= p.num_blocks) {
                                    report(p.status, PREFILL_ERR_BLOCK_TABLE);
                                    continue;
                                }
                                tma_store_4d(&tm_cache, src + ch * CHUNK + r * 128, ch * 64, it.g, 0, page * 2 + t);
                            }
                            if (lane < nst) bulk_commit();
                            // remaining rows one 16-byte unit per lane step
                            const int units = (rows - tma_rows) * 8 * L::NCH;
                            for (int x = lane; x < units; x += 32) {
                                const int rr = tma_rows + x / (8 * L::NCH);
                                const int ch = (x / 8) % L::NCH;
                                const int un = x % 8;
                                const int P_ = P0 + rr;
                                const int page = p.block_table[(size_t)it.i * p.mbps + P_ / bs];
                                if (page < 0 || page >= p.num_blocks) {
                                    report(p.status, PREFILL_ERR_BLOCK_TABLE);
                                    continue;
                                }
                                const uint4 val = *reinterpret_cast<const uint4 *>(
                                    gbase + (src - base) + ch * CHUNK + rr * 128 + ((un ^ (rr & 7)) << 4));
                                const size_t off =
                                    ((((size_t)page * 2 + t) * bs + P_ % bs) * G_ + it.g) * D + ch * 64 + un * 8;
                                *reinterpret_cast<uint4 *>(p.cache + off) = val;
                            }
                            if (lane < nst) bulk_wait_read0();  // each issuing lane waits for its own stores
                            __syncwarp();
                        }
                        if (lane == 0) mbar_arrive(bar(L::B_KVEMPTY + stage));
                        if (++stage == NST) { stage = 0; phase ^= 1; }
                    }
                }
            }
            bulk_wait0();  // every lane's stores complete before the kernel ends
            if (!ok && lane == 0) report(p.status, PREFILL_ERR_TIMEOUT);
            __syncwarp();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) tmem_dealloc(tmem, 512);
}

// Split-KV merge: a warp merges 32 consecutive packed rows x 32 columns of one
// query head, a lane per row (four warps per CTA, four heads; blockIdx.z picks
// the 32 columns).  A row's split count comes from part_nsp, written by this
// launch's attention kernel for every row of a valid sequence with the
// launch's epoch (a stale or unsplit row is left alone).  The loads of the
// splits' (max, sum) and of each 4-column chunk are 512 contiguous bytes per
// warp (the partials' chunk-major layout), all issued before any use; the
// lanes' rows then go through shared memory so that the output is written in
// 64-byte row pieces: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s with
// M = max_s m_s -- the merge rule the online softmax applies between blocks.
constexpr int kCombineWarps = 4;
constexpr int kMaxSplits = 8;
template <int D>
__global__ void __launch_bounds__(32 * kCombineWarps) combine_splits_kernel(const FwdParams p) {
    __shared__ __align__(16) uint16_t tile[kCombineWarps][32][40];  // 32 columns (+ 8: distinct banks)
    griddep_wait();  // the attention kernel's partials are complete
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y * kCombineWarps + warp;
    const int t0 = blockIdx.x * 32, t = t0 + lane, c0 = blockIdx.z * 8;  // 4-column chunks c0 .. c0 + 7
    if (h >= p.n_head) return;
    // every load that the launch's split count allows is issued before the
    // row's tag is known (speculative loads stay inside the workspace); the
    // splits' O chunks two at a time
    const bool in = t < p.total;
    const uint32_t tag = in ? p.part_nsp[t] : 0u;
    const float4 *po = reinterpret_cast<const float4 *>(p.part_o);
    auto oaddr = [&](int sp, int c) -> size_t {
        return (((size_t)sp * p.n_head + h) * (D / 4) + c0 + c) * p.total + t;
    };
    float2 ml[kMaxSplits];
#pragma unroll
    for (int sp = 0; sp < kMaxSplits; ++sp)
        if (in && sp < p.nsplit)
            ml[sp] = *reinterpret_cast<const float2 *>(p.part_ml + (((size_t)sp * p.n_head + h) * p.total + t) * 2);
    float4 f[2][8];
#pragma unroll
    for (int sp = 0; sp < 2; ++sp)
#pragma unroll
        for (int c = 0; c < 8; ++c)
            if (in && sp < p.nsplit) f[sp][c] = po[oaddr(sp, c)];
    int nsp = (in && (tag >> 4) == (p.epoch & 0x0fffffffu)) ? (int)(tag & 15u) : 0;  // else: not a row this launch split
    if (nsp > p.nsplit) nsp = p.nsplit;
    const bool mine = nsp > 1;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int sp = 0; sp < kMaxSplits; ++sp)
        if (mine && sp < nsp) M = fmaxf(M, ml[sp].x);
    float L = 0.f;
    float4 acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s0 = 0; s0 < kMaxSplits; s0 += 2) {
        if (s0 >= nsp) break;
        if (s0 > 0) {  // the next two splits (three or more splits: rare)
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    if (s0 + j < nsp) f[j][c] = po[oaddr(s0 + j, c)];
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            if (mine && s0 + j < nsp) {
                const float w = ex2(ml[s0 + j].x - M);
                L += w * ml[s0 + j].y;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    acc[c].x = fmaf(w, f[j][c].x, acc[c].x);
                    acc[c].y = fmaf(w, f[j][c].y, acc[c].y);
                    acc[c].z = fmaf(w, f[j][c].z, acc[c].z);
                    acc[c].w = fmaf(w, f[j][c].w, acc[c].w);
                }
            }
        }
    }
    const float inv = mine ? 1.f / L : 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint2 *>(&tile[warp][lane][4 * c]) =
            make_uint2(pack_bf16x2(acc[c].x * inv, acc[c].y * inv), pack_bf16x2(acc[c].z * inv, acc[c].w * inv));
    __syncwarp();
    // 64-byte row pieces: 4 lanes per row, 8 rows per store
    const uint32_t mask = __ballot_sync(0xffffffffu, mine);
#pragma unroll
    for (int rb = 0; rb < 32; rb += 8) {
        const int rr = rb + lane / 4, q = lane % 4;
        if ((mask >> rr) & 1u)
            *reinterpret_cast<uint4 *>(p.out + ((size_t)(t0 + rr) * p.n_head + h) * D + c0 * 4 + q * 8) =
                *reinterpret_cast<const uint4 *>(&tile[warp][rr][q * 8]);
    }
}

template <int D, int NST, bool F8 = false>
size_t smem_bytes(int P, int num_seqs) {
    return Lay<D, NST, F8>::SCHED + (size_t)(P + 1) * 12 + (((size_t)num_seqs * 2 + 15) & ~size_t(15)) + 1024;
}
constexpr size_t kMaxSmem = 227 * 1024;

// SM count of the current device, looked up once per device ordinal (a host
// may hold GPUs of different sizes; calls may come from several threads).
int sm_count() {
    static std::mutex mu;
    static std::map<int, int> by_device;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;
    }
    std::lock_guard<std::mutex> lock(mu);
    auto it = by_device.find(dev);
    if (it != by_device.end()) return it->second;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = 148;
    }
    by_device[dev] = n;
    return n;
}

template <int D, int NST, int MODE>
int launch_nst(const TensorMaps &maps, const FwdParams &p, void *stream) {
    const int P = cdiv(p.max_q, 2 * BM);
    const size_t smem = smem_bytes<D, NST, (MODE & kModeFp8) != 0>(P, p.num_seqs);
    cudaError_t e = cudaFuncSetAttribute(prefill_fwd_kernel<D, NST, MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return (int)e;
    const long long items_bound = (long long)p.num_seqs * p.n_head * P;
    const long long items = items_bound * (p.nsplit > 0 ? p.nsplit : 1);
    const int grid_s = (int)(items < sm_count() ? items : sm_count());
    // programmatic dependent launches: each kernel may be scheduled while the
    // one before it on the stream drains, and waits for it (griddep_wait)
    // before touching global memory
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid_s);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = (cudaStream_t)stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, prefill_fwd_kernel<D, NST, MODE>, maps.q, maps.k, maps.v, maps.cache, p, P);
    if (e != cudaSuccess || p.nsplit <= 1) return (int)e;
    cfg.gridDim = dim3((unsigned)cdiv(p.total, 32), (unsigned)cdiv(p.n_head, kCombineWarps), (unsigned)(D / 32));
    cfg.blockDim = dim3(32 * kCombineWarps);
    cfg.dynamicSmemBytes = 0;
    return (int)cudaLaunchKernelEx(&cfg, combine_splits_kernel<D>, p);
}

template <int D>
int launch(const TensorMaps &maps, const FwdParams &p, void *stream) {
    const int P = cdiv(p.max_q, 2 * BM);
    const bool nst5 = p.fp8 ? smem_bytes<D, 5, true>(P, p.num_seqs) <= kMaxSmem
                            : smem_bytes<D, 5>(P, p.num_seqs) <= kMaxSmem;
    const int mode = (p.window > 0 ? kModeWindow : 0) | (p.context_lens ? kModeChunk : 0) |
                     (p.cache ? 0 : kModeNoWrite) | (p.fp8 ? kModeFp8 : 0);
    switch (mode) {
        case 0: return nst5 ? launch_nst<D, 5, 0>(maps, p, stream) : launch_nst<D, 4, 0>(maps, p, stream);
        case 1: return nst5 ? launch_nst<D, 5, 1>(maps, p, stream) : launch_nst<D, 4, 1>(maps, p, stream);
        case 2: return nst5 ? launch_nst<D, 5, 2>(maps, p, stream) : launch_nst<D, 4, 2>(maps, p, stream);
        case 3: return nst5 ? launch_nst<D, 5, 3>(maps, p, stream) : launch_nst<D, 4, 3>(maps, p, stream);
        case kModeNoWrite:
            return nst5 ? launch_nst<D, 5, kModeNoWrite>(maps, p, stream)
                        : launch_nst<D, 4, kModeNoWrite>(maps, p, stream);
        case kModeChunk | kModeNoWrite | kModeFp8:
            return nst5 ? launch_nst<D, 5, kModeChunk | kModeNoWrite | kModeFp8>(maps, p, stream)
                        : launch_nst<D, 4, kModeChunk | kModeNoWrite | kModeFp8>(maps, p, stream);
        default: return (int)cudaErrorInvalidValue;  // no cache with a window or a prefix: not built
    }
}

}  // namespace

// Sizes the pipelined kernel handles (its schedule lives in shared memory).
bool fwd_pipelined_supported(const FwdParams &p, int head_dim) {
    const int P = cdiv(p.max_q, 2 * BM);
    if (P > 2048 || p.num_seqs > 4096) return false;
    const size_t smem = p.fp8 ? (head_dim == 64 ? smem_bytes<64, 4, true>(P, p.num_seqs)
                                                : smem_bytes<128, 4, true>(P, p.num_seqs))
                              : (head_dim == 64 ? smem_bytes<64, 4>(P, p.num_seqs) : smem_bytes<128, 4>(P, p.num_seqs));
    return smem <= kMaxSmem;
}

// Fixed cost of splitting (the partial writes and the merge kernel), in units
// of one kv block step of a work item: the merge path of a 512-row chunk of an
// 8k GQA prompt takes ~6 us (release of the merge launch, merging, release of
// the next launch) against ~2 us per step; on the 16 chunks of that prompt a
// cost of 4 steps ran fastest (6: 0.859 ms, 4: 0.851, 3: 0.858, 2: 0.863).
constexpr double kSplitCostSteps = 4.0;

int device_sm_count() { return sm_count(); }

int fwd_choose_splits(const FwdParams &p) {
    // Split only when the call has fewer work items than SMs: pick the split
    // count (up to 8) that minimises waves x blocks per split + the split's
    // fixed cost, keeping >= kMinSplitBlocks blocks per split of the longest
    // kv range.
    const long long items = (long long)p.num_seqs * p.n_head * cdiv(p.max_q, 2 * BM);
    const int sms = sm_count();
    if (items <= 0 || items >= sms) return 1;
    int nk = cdiv(p.max_ctx, BN) + cdiv(p.max_q, BN);
    if (p.window > 0) nk = imin(nk, cdiv(p.window, BN) + 2);  // a windowed query block's range
    int best = 1;
    double best_cost = (double)nk;  // one wave of whole ranges
    for (int sp = 2; sp <= kMaxSplits; ++sp) {
        if (nk / sp < kMinSplitBlocks) break;
        const double waves = (double)((items * sp + sms - 1) / sms);
        const double cost = waves * cdiv(nk, sp) + kSplitCostSteps;
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = sp;
        }
    }
    return best;
}

size_t fwd_split_workspace_bytes(const FwdParams &p, int head_dim) {
    if (p.nsplit <= 1) return 0;
    return (size_t)p.nsplit * p.total * p.n_head * ((size_t)head_dim + 2) * sizeof(float) +
           (size_t)p.total * sizeof(uint32_t);
}

namespace {
// y[i] = exp2_fma2(x[i]) for a test of the polynomial against exp2 (one pair per thread).
__global__ void exp2_fma2_probe_kernel(const float *x, float *y, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
    float ra, rb;
    exp2_fma2(a, b, ra, rb);
    y[i] = ra;
    if (i + 1 < n) y[i + 1] = rb;
}
}  // namespace

int launch_exp2_fma2_probe(const float *x, float *y, int n, void *stream) {
    if (n <= 0) return 0;
    const int pairs = (n + 1) / 2;
    exp2_fma2_probe_kernel<<<(pairs + 255) / 256, 256, 0, (cudaStream_t)stream>>>(x, y, n);
    return (int)cudaGetLastError();
}

int launch_fwd(const TensorMaps &maps, const FwdParams &p, int head_dim, void *stream) {
    if (head_dim == 64) return launch<64>(maps, p, stream);
    return launch<128>(maps, p, stream);
}

}  // namespace pf
