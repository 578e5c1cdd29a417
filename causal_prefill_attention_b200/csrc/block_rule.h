// block_rule.h -- the causal block rule of the tiled attention
// (hncyxsy.com/news/270449 §4.3): a kv block entirely after a query block is
// never issued, a kv block entirely before it needs no mask, and the block on
// the diagonal is masked by column inside the block.  With chunked prefill
// (hncyxsy.com/news/227904 §2.1) the cached prefix comes first: every chunk
// row sees all of it, so prefix blocks are unmasked except for the columns
// past the end of the prefix.
//
// Sliding window (lnwmold.com/news/496245 §4.1): with a window of W keys, row
// P sees keys P-W+1 .. P only.  The blocks a query block needs are still one
// contiguous run, now starting at the block that holds its first row's lowest
// key, and a block is also masked from below (columns < col_lo(r)) where the
// window's edge crosses it.  W <= 0 means no window.
//
// One header for the kernels and the host-side export, so the rule tested on
// the host is the rule the device runs.
#pragma once

#if defined(__CUDACC__)
#define PF_HD __host__ __device__ __forceinline__
#else
#define PF_HD inline
#endif

namespace pf {

PF_HD int cdiv(int a, int b) { return (a + b - 1) / b; }
PF_HD int imin(int a, int b) { return a < b ? a : b; }
PF_HD int imax(int a, int b) { return a > b ? a : b; }

// Number of kv blocks a query block qb (rows [qb*bm, qb*bm+bm) of a chunk of
// n rows that follows ctx cached tokens) must visit without a window: prefix
// blocks first, then the chunk's own blocks up to the one holding the block's
// last valid row.  Under a window the visit starts at first_kv_block and still
// ends here.
PF_HD int num_kv_blocks(int qb, int ctx, int n, int bm, int bn) {
    int a0 = qb * bm;
    if (a0 >= n || a0 < 0) return 0;
    int a_max = imin(a0 + bm, n) - 1;
    return cdiv(ctx, bn) + a_max / bn + 1;
}

// Lowest absolute key position visible to row r of query block qb under a
// window of `window` keys (may be negative: then nothing is cut).
PF_HD long long window_low_key(int qb, int r, int ctx, int bm, int window) {
    return (long long)ctx + (long long)qb * bm + r - window + 1;
}

// First kv block query block qb visits: the block holding its first row's
// lowest visible key (0 without a window).
PF_HD int first_kv_block(int qb, int ctx, int n, int bm, int bn, int window) {
    if (window <= 0 || qb * bm >= n) return 0;
    const long long lo = window_low_key(qb, 0, ctx, bm, window);
    if (lo <= 0) return 0;
    if (lo < ctx) return (int)(lo / bn);
    return cdiv(ctx, bn) + (int)((lo - ctx) / bn);
}

// Block j of query block qb: key range start (absolute position), and whether
// every valid (row, key) pair of the block is visible.  For a masked block row
// r sees the columns [col_lo(r), col_limit(r)).
struct KvBlock {
    int key_begin;   // absolute position of column 0
    int prefix;      // 1: keys come from the cache; 0: from this call's k/v rows
    int src_row;     // prefix: first position (== key_begin); chunk: chunk-local row of column 0
    int full;        // 1: no column is masked for any valid row
    int lim_const;   // prefix: columns < lim_const are visible (same for all rows)
    int diag_off;    // chunk: row r sees columns c <= r + diag_off ...
    int lim_n;       // ... and c < lim_n (end of the chunk)
    int lo_off;      // window: row r sees columns c >= r + lo_off (very negative without a window)
};

PF_HD KvBlock kv_block(int qb, int j, int ctx, int n, int bm, int bn, int window) {
    KvBlock b;
    int np = cdiv(ctx, bn);
    if (j < np) {
        b.prefix = 1;
        b.key_begin = j * bn;
        b.src_row = j * bn;
        b.lim_const = imin(bn, ctx - j * bn);
        b.full = b.lim_const == bn;
        b.diag_off = bn;   // unused for prefix blocks
        b.lim_n = bn;
    } else {
        int jc = j - np;
        b.prefix = 0;
        b.key_begin = ctx + jc * bn;
        b.src_row = jc * bn;
        b.lim_const = bn;
        // row r is chunk row a = qb*bm + r; column c is chunk key jc*bn + c;
        // visible iff jc*bn + c <= a and jc*bn + c < n.
        b.diag_off = qb * bm - jc * bn;
        b.lim_n = n - jc * bn;
        b.full = (b.diag_off + 1 >= bn) && (b.lim_n >= bn);
    }
    if (window > 0) {
        // column c of row r is position key_begin + c; visible iff it is at
        // least the row's lowest key.  The block stays unmasked only if even
        // the last valid row sees column 0.
        const long long off = window_low_key(qb, 0, ctx, bm, window) - b.key_begin;
        b.lo_off = off < -(1 << 29) ? -(1 << 29) : (off > (1 << 29) ? (1 << 29) : (int)off);
        const int r_last = imin(bm, n - qb * bm) - 1;
        if (r_last + b.lo_off > 0) b.full = 0;
    } else {
        b.lo_off = -(1 << 29);
    }
    return b;
}

// Visible columns of row r in block b: [col_lo, col_limit), each clamped to [0, bn].
PF_HD int col_limit(const KvBlock &b, int r, int bn) {
    if (b.prefix) return b.lim_const;
    int lim = imin(r + b.diag_off + 1, b.lim_n);
    return imax(0, imin(lim, bn));
}

PF_HD int col_lo(const KvBlock &b, int r, int bn) { return imax(0, imin(r + b.lo_off, bn)); }

}  // namespace pf
