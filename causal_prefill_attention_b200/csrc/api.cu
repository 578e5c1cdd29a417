// api.cu -- the C ABI of libprefill (include/prefill.h): host-side argument
// checks, TMA tensor-map encoding, kernel launch.  Allocates no device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <cstdint>
#include <atomic>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "../../include/prefill.h"
#include "block_rule.h"
#include "decode.h"
#include "params.h"
#include "qkv_gemm.h"

namespace {

using EncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeFn encode_fn() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(ptr);
    });
    return fn;
}

// bf16 tensor map with 128-byte swizzle; dims innermost first, strides in bytes
// for dims 1..rank-1.  Out-of-range boxes are filled with zeros.
bool encode(CUtensorMap *m, const void *ptr, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
            const cuuint32_t *box) {
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// uint8 tensor map (e4m3 codes) without swizzle: rows land as plain bytes.
bool encode_u8(CUtensorMap *m, const void *ptr, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
               const cuuint32_t *box) {
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, (cuuint32_t)rank, const_cast<void *>(ptr), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// uint8 tensor map with 128-byte swizzle (e4m3 codes in 128-byte rows).
bool encode_u8_sw128(CUtensorMap *m, const void *ptr, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
                     const cuuint32_t *box) {
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, (cuuint32_t)rank, const_cast<void *>(ptr), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Decode runs the whole-page kernel where it applies unless
// LIBPREFILL_DECODE=warp selects the per-warp kernel (used to compare the two
// on the same inputs).
bool use_whole_page_decode() {
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("LIBPREFILL_DECODE");
        v = (e && std::strcmp(e, "warp") == 0) ? 0 : 1;
    }
    return v == 1;
}

// The pipelined kernel runs unless LIBPREFILL_KERNEL=simple selects the
// one-CTA-per-block kernel (used to compare the two on the same inputs).
bool use_pipelined() {
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("LIBPREFILL_KERNEL");
        v = (e && std::strcmp(e, "simple") == 0) ? 0 : 1;
    }
    return v == 1;
}

std::atomic<int> g_test_stall{0};
// Launch counter: tags the rows a launch splits, so that the merge kernel never
// takes another launch's leftovers in a reused workspace for its own.
std::atomic<uint32_t> g_epoch{1};

// Device workspaces: one buffer per (device, stream, kind), allocated on the
// first call that needs it and grown when a larger call needs more.  Kept for
// later calls; a separate buffer per stream keeps concurrent streams apart.
// Kinds: the split-KV partials, and the staging of a chunked prefill over an
// FP8 cache (which then also uses the split-KV partials).
//
// Growth is stream-ordered (cudaFreeAsync of the old buffer, cudaMallocAsync of
// the new one, both on the call's stream): the old buffer is released only
// after the work already queued on the stream that reads it, and the host never
// waits.  A caller that cannot let the library allocate at all uses
// prefill_attn_chunked_noalloc.
enum WorkspaceKind { kSplitPartials = 0, kFp8Staging = 1 };
struct Workspace {
    void *ptr = nullptr;
    size_t bytes = 0;
};
std::mutex g_ws_mu;
std::map<std::tuple<int, void *, int>, Workspace> g_ws;

void *device_workspace(int kind, size_t bytes, void *stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    std::lock_guard<std::mutex> lock(g_ws_mu);
    Workspace &w = g_ws[std::make_tuple(dev, stream, kind)];
    if (w.bytes < bytes) {
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        if (w.ptr) {
            cudaFreeAsync(w.ptr, st);  // after the queued work that reads it
            w.ptr = nullptr;
            w.bytes = 0;
        }
        // round up so that slowly growing calls do not reallocate every time
        const size_t want = bytes + bytes / 4;
        if (cudaMallocAsync(&w.ptr, want, st) != cudaSuccess) {
            cudaGetLastError();
            w.ptr = nullptr;
            return nullptr;
        }
        w.bytes = want;
    }
    return w.ptr;
}

void *split_workspace(size_t bytes, void *stream) { return device_workspace(kSplitPartials, bytes, stream); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace pf {

int run_prefill(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v, int total, const int32_t *cu,
                const int32_t *ctx_lens, bool chunked, int num_seqs, int max_q, long long max_ctx, int n_head,
                int n_kv_head, int head_dim, float scale, prefill_bf16 *out, prefill_bf16 *cache, int num_blocks,
                const int32_t *bt, int mbps, int bs, int32_t *status, prefill_stream_t stream, void *scratch,
                size_t scratch_bytes, int window, uint8_t *cache8, const float *k_scale, const float *v_scale,
                const float *k_fold, const float *v_fold) {
    if (!q || !k || !v || !cu || !out || !(cache || cache8) || !bt || (chunked && !ctx_lens)) return PREFILL_ERR_NULL;
    if (cache8 && (!k_scale || !v_scale)) return PREFILL_ERR_NULL;
    if (cache8 && (cache || window > 0)) return PREFILL_ERR_UNSUPPORTED;
    // chunked over an FP8 cache: every key and value the chunk attends to is a
    // cache value, the scales folded into the kernel's scores and output
    const bool fp8_chunk = cache8 && chunked;
    if (fp8_chunk) {
        k_fold = k_scale;
        v_fold = v_scale;
    }
    if (total < 0 || num_seqs < 0 || max_q < 0 || max_ctx < 0) return PREFILL_ERR_SHAPE;
    if (n_head < 1 || n_kv_head < 1 || n_head % n_kv_head != 0) return PREFILL_ERR_SHAPE;
    if (head_dim != 64 && head_dim != 128) return PREFILL_ERR_UNSUPPORTED;
    if (bs != 16 && bs != 32 && bs != 64 && bs != 128) return PREFILL_ERR_UNSUPPORTED;
    if (!(std::isfinite(scale) && scale > 0.f)) return PREFILL_ERR_UNSUPPORTED;
    if (window < 0) return PREFILL_ERR_SHAPE;
    if (num_blocks < 1 || mbps < 1) return PREFILL_ERR_BLOCK_TABLE;
    // each bound must fit the table; the exact per-sequence check (context +
    // chunk length) runs on the device, where the lengths are
    if (max_ctx > (long long)mbps * bs || max_q > (long long)mbps * bs) return PREFILL_ERR_BLOCK_TABLE;
    if (num_seqs > 65535 || n_head > 65535) return PREFILL_ERR_UNSUPPORTED;
    if ((long long)num_blocks * 2 * bs * n_kv_head * head_dim > (1ll << 40)) return PREFILL_ERR_SHAPE;
    const void *pool = cache ? static_cast<const void *>(cache) : static_cast<const void *>(cache8);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(pool))
        return PREFILL_ERR_ALIGNMENT;
    if (total == 0 || num_seqs == 0 || max_q == 0) return PREFILL_OK;
    if (fp8_chunk && (!use_pipelined() || (long long)total * n_kv_head * head_dim > (1ll << 40)))
        return PREFILL_ERR_UNSUPPORTED;

    // FP8 chunk: its codes go to the pool (the attention reads them back as the
    // chunk's own keys and values) and into a dense copy [total][G][D] of the
    // call's rows, from which the kernel loads its own tiles by TMA
    uint8_t *k8 = nullptr, *v8 = nullptr;
    if (fp8_chunk) {
        const size_t rowb = (size_t)n_kv_head * head_dim;
        char *ws = static_cast<char *>(device_workspace(kFp8Staging, 2 * (size_t)total * rowb, stream));
        if (!ws) return PREFILL_ERR_CUDA;
        k8 = reinterpret_cast<uint8_t *>(ws);
        v8 = reinterpret_cast<uint8_t *>(ws + (size_t)total * rowb);
    }

    pf::TensorMaps maps;
    const cuuint64_t D = head_dim, H = n_head, G = n_kv_head, T = total;
    // q / k / v: {64 columns, head, token, 64-column chunk}; the chunk is the
    // outermost dimension (stride 128 B), so one box {64, 1, 128, D/64} lands a
    // whole 128-row tile chunk-major: D/64 blocks of 128 rows x 128 B, each
    // 128-byte swizzled -- the layout the MMA descriptors expect.
    const cuuint64_t NCH = D / 64;
    {
        const cuuint64_t dims[4] = {64, H, T, NCH}, strides[3] = {D * 2, H * D * 2, 128};
        const cuuint32_t box[4] = {64, 1, 128, (cuuint32_t)NCH};
        if (!encode(&maps.q, q, 4, dims, strides, box)) return PREFILL_ERR_CUDA;
    }
    if (fp8_chunk) {
        // dense codes {D bytes, head, token, 1}, box {D, 1, 128, 1}: a tile's rows as plain bytes
        const cuuint64_t dims[4] = {D, G, T, 1}, strides[3] = {D, G * D, T * G * D};
        const cuuint32_t box[4] = {(cuuint32_t)D, 1, 128, 1};
        if (!encode_u8(&maps.k, k8, 4, dims, strides, box)) return PREFILL_ERR_CUDA;
        if (!encode_u8(&maps.v, v8, 4, dims, strides, box)) return PREFILL_ERR_CUDA;
    } else {
        const cuuint64_t dims[4] = {64, G, T, NCH}, strides[3] = {D * 2, G * D * 2, 128};
        const cuuint32_t box[4] = {64, 1, 128, (cuuint32_t)NCH};
        if (!encode(&maps.k, k, 4, dims, strides, box)) return PREFILL_ERR_CUDA;
        if (!encode(&maps.v, v, 4, dims, strides, box)) return PREFILL_ERR_CUDA;
    }
    if (fp8_chunk) {
        // the FP8 pool {D bytes, head, slot, page * 2 + K/V}, box {D, 1, bs, 1}: one whole page
        const cuuint64_t dims[4] = {D, G, (cuuint64_t)bs, (cuuint64_t)num_blocks * 2};
        const cuuint64_t strides[3] = {D, G * D, (cuuint64_t)bs * G * D};
        const cuuint32_t box[4] = {(cuuint32_t)D, 1, (cuuint32_t)bs, 1};
        if (!encode_u8(&maps.cache, cache8, 4, dims, strides, box)) return PREFILL_ERR_CUDA;
    } else if (cache) {
        const cuuint64_t dims[4] = {D, G, (cuuint64_t)bs, (cuuint64_t)num_blocks * 2};
        const cuuint64_t strides[3] = {D * 2, G * D * 2, (cuuint64_t)bs * G * D * 2};
        const cuuint32_t box[4] = {64, 1, (cuuint32_t)bs, 1};
        if (!encode(&maps.cache, cache, 4, dims, strides, box)) return PREFILL_ERR_CUDA;
    } else {
        maps.cache = maps.k;  // a valid map the FP8 kernels never use
    }

    pf::FwdParams p;
    p.k = k;
    p.v = v;
    p.out = out;
    p.cache = cache;
    p.cu_seqlens = cu;
    p.context_lens = chunked ? ctx_lens : nullptr;
    p.block_table = bt;
    p.status = status;
    p.num_seqs = num_seqs;
    p.n_head = n_head;
    p.n_kv_head = n_kv_head;
    p.group = n_head / n_kv_head;
    p.total = total;
    p.num_blocks = num_blocks;
    p.mbps = mbps;
    p.block_size = bs;
    p.max_q = max_q;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.test_stall = g_test_stall.exchange(0);
    p.max_ctx = (int)max_ctx;
    p.window = window;
    p.nsplit = 1;
    p.part_o = nullptr;
    p.part_ml = nullptr;
    p.part_nsp = nullptr;
    p.epoch = g_epoch.fetch_add(1) & 0x0fffffffu;
    p.k_fold = k_fold;
    p.v_fold = v_fold;
    p.fp8 = fp8_chunk ? 1 : 0;

    int e;
    const bool pipelined = use_pipelined() && pf::fwd_pipelined_supported(p, head_dim);
    // the FP8 write and the folded scales live in the pipelined kernel only
    if ((cache8 || k_fold || v_fold) && !pipelined) return PREFILL_ERR_UNSUPPORTED;
    auto store_fp8 = [&](const int32_t *ctxs, uint8_t *dk8, uint8_t *dv8) -> int {
        pf::Fp8StoreParams sp;
        sp.k = k;
        sp.v = v;
        sp.cu_seqlens = cu;
        sp.context_lens = ctxs;
        sp.k_scale = k_scale;
        sp.v_scale = v_scale;
        sp.cache8 = cache8;
        sp.dense_k8 = dk8;
        sp.dense_v8 = dv8;
        sp.block_table = bt;
        sp.status = status;
        sp.total = total;
        sp.num_seqs = num_seqs;
        sp.n_kv_head = n_kv_head;
        sp.num_blocks = num_blocks;
        sp.mbps = mbps;
        sp.block_size = bs;
        return pf::launch_kv_store_fp8(sp, head_dim, stream);
    };
    if (pipelined) {
        p.nsplit = pf::fwd_choose_splits(p);
        // caller-supplied scratch of a fixed size: the largest split count whose
        // partials fit it (1 needs none), so every call still runs
        while (scratch && p.nsplit > 1 && pf::fwd_split_workspace_bytes(p, head_dim) > scratch_bytes) --p.nsplit;
        if (p.nsplit > 1) {
            const size_t o_bytes = (size_t)p.nsplit * p.total * p.n_head * head_dim * sizeof(float);
            const size_t need = pf::fwd_split_workspace_bytes(p, head_dim);
            char *ws = static_cast<char *>(scratch ? scratch : split_workspace(need, stream));
            if (ws) {
                p.part_o = reinterpret_cast<float *>(ws);
                p.part_ml = reinterpret_cast<float *>(ws + o_bytes);
                p.part_nsp = reinterpret_cast<uint32_t *>(ws + o_bytes +
                                                          (size_t)p.nsplit * p.total * p.n_head * 2 * sizeof(float));
            } else {
                p.nsplit = 1;  // no workspace: run unsplit
            }
        }
        // FP8 chunk: the chunk's codes are stored first (the kernel reads them back)
        e = fp8_chunk ? store_fp8(ctx_lens, k8, v8) : 0;
        if (e == 0) e = pf::launch_fwd(maps, p, head_dim, stream);
        if (e == 0 && cache8 && !fp8_chunk) {
            // FP8 cache of a whole prompt: quantize this call's K/V rows into their
            // slots after the attention (over the bf16 inputs).  A separate pass:
            // quantizing inside the attention kernel (by its spare warps, from L2)
            // measured slower than this launch.
            e = store_fp8(nullptr, nullptr, nullptr);
        }
    } else {
        e = pf::launch_fwd_v0(maps, p, head_dim, stream);
    }
    return e == 0 ? PREFILL_OK : PREFILL_ERR_CUDA;
}

}  // namespace pf

extern "C" {

int prefill_attn(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v, int total_tokens,
                 const int32_t *cu_seqlens, int num_seqs, int max_seqlen, int n_head, int n_kv_head, int head_dim,
                 float scale, prefill_bf16 *out, prefill_bf16 *kv_cache, int num_blocks,
                 const int32_t *block_table, int max_blocks_per_seq, int block_size, int32_t *status_dev,
                 prefill_stream_t stream) {
    return pf::run_prefill(q, k, v, total_tokens, cu_seqlens, nullptr, false, num_seqs, max_seqlen, 0, n_head,
                           n_kv_head, head_dim, scale, out, kv_cache, num_blocks, block_table, max_blocks_per_seq,
                           block_size, status_dev, stream, nullptr, 0);
}

int prefill_attn_chunked(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v, int total_q,
                         const int32_t *cu_seqlens_q, const int32_t *context_lens, int num_seqs, int max_q_len,
                         int max_context_len, int n_head, int n_kv_head, int head_dim, float scale,
                         prefill_bf16 *out, prefill_bf16 *kv_cache, int num_blocks, const int32_t *block_table,
                         int max_blocks_per_seq, int block_size, int32_t *status_dev, prefill_stream_t stream) {
    return pf::run_prefill(q, k, v, total_q, cu_seqlens_q, context_lens, true, num_seqs, max_q_len, max_context_len,
                           n_head, n_kv_head, head_dim, scale, out, kv_cache, num_blocks, block_table,
                           max_blocks_per_seq, block_size, status_dev, stream, nullptr, 0);
}

int prefill_attn_fp8_cache(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v, int total_tokens,
                           const int32_t *cu_seqlens, int num_seqs, int max_seqlen, int n_head, int n_kv_head,
                           int head_dim, float scale, const float *k_scale, const float *v_scale, prefill_bf16 *out,
                           uint8_t *kv_cache_fp8, int num_blocks, const int32_t *block_table,
                           int max_blocks_per_seq, int block_size, int32_t *status_dev, prefill_stream_t stream) {
    if (!kv_cache_fp8) return PREFILL_ERR_NULL;
    return pf::run_prefill(q, k, v, total_tokens, cu_seqlens, nullptr, false, num_seqs, max_seqlen, 0, n_head,
                           n_kv_head, head_dim, scale, out, nullptr, num_blocks, block_table, max_blocks_per_seq,
                           block_size, status_dev, stream, nullptr, 0, 0, kv_cache_fp8, k_scale, v_scale);
}

int prefill_attn_chunked_fp8(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v, int total_q,
                             const int32_t *cu_seqlens_q, const int32_t *context_lens, int num_seqs, int max_q_len,
                             int max_context_len, int n_head, int n_kv_head, int head_dim, float scale,
                             const float *k_scale, const float *v_scale, prefill_bf16 *out, uint8_t *kv_cache_fp8,
                             int num_blocks, const int32_t *block_table, int max_blocks_per_seq, int block_size,
                             int32_t *status_dev, prefill_stream_t stream) {
    if (!kv_cache_fp8 || !context_lens) return PREFILL_ERR_NULL;
    return pf::run_prefill(q, k, v, total_q, cu_seqlens_q, context_lens, true, num_seqs, max_q_len, max_context_len,
                           n_head, n_kv_head, head_dim, scale, out, nullptr, num_blocks, block_table,
                           max_blocks_per_seq, block_size, status_dev, stream, nullptr, 0, 0, kv_cache_fp8, k_scale,
                           v_scale);
}

int prefill_attn_sliding_window(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v, int total_q,
                                const int32_t *cu_seqlens_q, const int32_t *context_lens, int num_seqs,
                                int max_q_len, int max_context_len, int n_head, int n_kv_head, int head_dim,
                                float scale, int window, prefill_bf16 *out, prefill_bf16 *kv_cache, int num_blocks,
                                const int32_t *block_table, int max_blocks_per_seq, int block_size,
                                int32_t *status_dev, prefill_stream_t stream) {
    if (window < 1) return PREFILL_ERR_SHAPE;
    if (!context_lens && max_context_len != 0) return PREFILL_ERR_SHAPE;
    return pf::run_prefill(q, k, v, total_q, cu_seqlens_q, context_lens, context_lens != nullptr, num_seqs,
                           max_q_len, max_context_len, n_head, n_kv_head, head_dim, scale, out, kv_cache,
                           num_blocks, block_table, max_blocks_per_seq, block_size, status_dev, stream, nullptr, 0,
                           window);
}

}  // extern "C"

namespace {

// Shared body of paged_decode_attn (bf16 cache) and paged_decode_attn_fp8
// (e4m3 cache with per-kv-head scales).
int run_decode(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v, const int32_t *context_lens,
               int num_seqs, int max_context_len, int n_head, int n_kv_head, int head_dim, float scale,
               prefill_bf16 *out, void *kv_cache, bool fp8, const float *k_scale, const float *v_scale,
               int num_blocks, const int32_t *block_table, int max_blocks_per_seq, int block_size,
               int32_t *status_dev, prefill_stream_t stream) {
    if (!q || !k || !v || !context_lens || !out || !kv_cache || !block_table) return PREFILL_ERR_NULL;
    if (fp8 && (!k_scale || !v_scale)) return PREFILL_ERR_NULL;
    if (num_seqs < 0 || max_context_len < 0) return PREFILL_ERR_SHAPE;
    if (n_head < 1 || n_kv_head < 1 || n_head % n_kv_head != 0) return PREFILL_ERR_SHAPE;
    if (n_head / n_kv_head > 16) return PREFILL_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PREFILL_ERR_UNSUPPORTED;
    if (block_size != 16 && block_size != 32 && block_size != 64 && block_size != 128) return PREFILL_ERR_UNSUPPORTED;
    if (!(std::isfinite(scale) && scale > 0.f)) return PREFILL_ERR_UNSUPPORTED;
    if (num_blocks < 1 || max_blocks_per_seq < 1) return PREFILL_ERR_BLOCK_TABLE;
    if ((long long)max_context_len + 1 > (long long)max_blocks_per_seq * block_size) return PREFILL_ERR_BLOCK_TABLE;
    if (num_seqs > pf::kDecodeMaxSeqs || n_kv_head > 65535) return PREFILL_ERR_UNSUPPORTED;
    if ((long long)num_blocks * 2 * block_size * n_kv_head * head_dim > (1ll << 40)) return PREFILL_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(kv_cache))
        return PREFILL_ERR_ALIGNMENT;
    if (num_seqs == 0) return PREFILL_OK;

    pf::DecodeParams p;
    p.q = q;
    p.k = k;
    p.v = v;
    p.out = out;
    p.cache = fp8 ? nullptr : static_cast<prefill_bf16 *>(kv_cache);
    p.context_lens = context_lens;
    p.block_table = block_table;
    p.status = status_dev;
    p.num_seqs = num_seqs;
    p.n_head = n_head;
    p.n_kv_head = n_kv_head;
    p.num_blocks = num_blocks;
    p.mbps = max_blocks_per_seq;
    p.block_size = block_size;
    p.max_ctx = max_context_len;
    p.keys_per_unit = pf::decode_keys_per_unit(max_context_len);
    p.max_units = pf::cdiv(max_context_len + 1, p.keys_per_unit);
    p.scale_log2 = scale * 1.4426950408889634f;
    p.part_o = nullptr;
    p.part_ml = nullptr;
    p.cache8 = fp8 ? static_cast<uint8_t *>(kv_cache) : nullptr;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    if (n_kv_head % 8 == 0 && (!fp8 || head_dim == 128) && use_whole_page_decode()) {
        // the cache as [page * 2 + t][kv head][position][column] (innermost last):
        // a box of 16 positions x 8 kv heads x 128 bytes is one step of one slab
        const cuuint64_t es = fp8 ? 1 : 2;
        const cuuint64_t dims[4] = {(cuuint64_t)head_dim, (cuuint64_t)block_size, (cuuint64_t)n_kv_head,
                                    2 * (cuuint64_t)num_blocks};
        const cuuint64_t strides[3] = {(cuuint64_t)n_kv_head * head_dim * es, (cuuint64_t)head_dim * es,
                                       (cuuint64_t)block_size * n_kv_head * head_dim * es};
        const cuuint32_t box[4] = {fp8 ? 128u : 64u, 16u, 8u, 1u};
        CUtensorMap tm;
        const bool enc = fp8 ? encode_u8_sw128(&tm, kv_cache, 4, dims, strides, box)
                             : encode(&tm, kv_cache, 4, dims, strides, box);
        if (!enc) return PREFILL_ERR_CUDA;
        p.grid = pf::device_sm_count();
        // partial rows [piece id][n_head / slabs] (fp32 O, then max and sum), then
        // the [num_seqs + 1] step scan, in the split-KV partials' workspace
        const size_t rows = (size_t)p.grid * (n_head / (n_kv_head / 8)) + (size_t)num_seqs * n_head;
        const size_t fbytes = rows * ((size_t)head_dim + 2) * sizeof(float);
        char *ws = static_cast<char *>(split_workspace(fbytes + ((size_t)num_seqs + 1) * sizeof(int32_t), stream));
        if (!ws) return PREFILL_ERR_CUDA;
        p.part_o = reinterpret_cast<float *>(ws);
        p.part_ml = reinterpret_cast<float *>(ws + rows * head_dim * sizeof(float));
        p.seg_cum = reinterpret_cast<int32_t *>(ws + fbytes);
        return pf::launch_decode_tma(p, &tm, head_dim, fp8, stream) == 0 ? PREFILL_OK : PREFILL_ERR_CUDA;
    }
    if (p.max_units > 1) {
        // partials [max_units][num_seqs][n_head][head_dim + 2] fp32, in the same
        // per-(device, stream) workspace as the prefill split-KV partials
        const size_t rows = (size_t)p.max_units * num_seqs * n_head;
        char *ws = static_cast<char *>(split_workspace(rows * ((size_t)head_dim + 2) * sizeof(float), stream));
        if (!ws) return PREFILL_ERR_CUDA;
        p.part_o = reinterpret_cast<float *>(ws);
        p.part_ml = reinterpret_cast<float *>(ws + rows * head_dim * sizeof(float));
    }
    return pf::launch_decode(p, head_dim, fp8, stream) == 0 ? PREFILL_OK : PREFILL_ERR_CUDA;
}

}  // namespace

extern "C" {

int paged_decode_attn(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v,
                      const int32_t *context_lens, int num_seqs, int max_context_len, int n_head, int n_kv_head,
                      int head_dim, float scale, prefill_bf16 *out, prefill_bf16 *kv_cache, int num_blocks,
                      const int32_t *block_table, int max_blocks_per_seq, int block_size, int32_t *status_dev,
                      prefill_stream_t stream) {
    return run_decode(q, k, v, context_lens, num_seqs, max_context_len, n_head, n_kv_head, head_dim, scale, out,
                      kv_cache, false, nullptr, nullptr, num_blocks, block_table, max_blocks_per_seq, block_size,
                      status_dev, stream);
}

int paged_decode_attn_fp8(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v,
                          const int32_t *context_lens, int num_seqs, int max_context_len, int n_head, int n_kv_head,
                          int head_dim, float scale, const float *k_scale, const float *v_scale, prefill_bf16 *out,
                          uint8_t *kv_cache_fp8, int num_blocks, const int32_t *block_table, int max_blocks_per_seq,
                          int block_size, int32_t *status_dev, prefill_stream_t stream) {
    return run_decode(q, k, v, context_lens, num_seqs, max_context_len, n_head, n_kv_head, head_dim, scale, out,
                      kv_cache_fp8, true, k_scale, v_scale, num_blocks, block_table, max_blocks_per_seq, block_size,
                      status_dev, stream);
}

int kv_cache_store_fp8(const prefill_bf16 *k, const prefill_bf16 *v, int total_tokens, const int32_t *cu_seqlens,
                       const int32_t *context_lens, int num_seqs, int n_kv_head, int head_dim, const float *k_scale,
                       const float *v_scale, uint8_t *kv_cache_fp8, int num_blocks, const int32_t *block_table,
                       int max_blocks_per_seq, int block_size, int32_t *status_dev, prefill_stream_t stream) {
    if (!k || !v || !cu_seqlens || !k_scale || !v_scale || !kv_cache_fp8 || !block_table) return PREFILL_ERR_NULL;
    if (total_tokens < 0 || num_seqs < 0 || n_kv_head < 1) return PREFILL_ERR_SHAPE;
    if (head_dim != 64 && head_dim != 128) return PREFILL_ERR_UNSUPPORTED;
    if (block_size != 16 && block_size != 32 && block_size != 64 && block_size != 128) return PREFILL_ERR_UNSUPPORTED;
    if (num_blocks < 1 || max_blocks_per_seq < 1) return PREFILL_ERR_BLOCK_TABLE;
    if (!aligned16(k) || !aligned16(v) || !aligned16(kv_cache_fp8)) return PREFILL_ERR_ALIGNMENT;
    if (total_tokens == 0 || num_seqs == 0) return PREFILL_OK;
    pf::Fp8StoreParams p;
    p.k = k;
    p.v = v;
    p.cu_seqlens = cu_seqlens;
    p.context_lens = context_lens;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.cache8 = kv_cache_fp8;
    p.block_table = block_table;
    p.status = status_dev;
    p.total = total_tokens;
    p.num_seqs = num_seqs;
    p.n_kv_head = n_kv_head;
    p.num_blocks = num_blocks;
    p.mbps = max_blocks_per_seq;
    p.block_size = block_size;
    return pf::launch_kv_store_fp8(p, head_dim, stream) == 0 ? PREFILL_OK : PREFILL_ERR_CUDA;
}

}  // extern "C"

namespace {

// y = x w^T on the tcgen05 GEMM: x [M][K], w [N][K] (bf16, K-contiguous), the
// output columns routed by p (Q | K | V ranges, or one plain output).
int run_linear(const prefill_bf16 *x, const prefill_bf16 *w, int M, int K, int N, pf::QkvParams &p,
               prefill_stream_t stream) {
    CUtensorMap tm_x, tm_w;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M}, strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {64, 128};
        if (!encode(&tm_x, x, 2, dims, strides, box)) return PREFILL_ERR_CUDA;
    }
    const int tile_n = pf::qkv_gemm_tile_n(M, N, pf::device_sm_count());
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N}, strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {64, (cuuint32_t)tile_n};
        if (!encode(&tm_w, w, 2, dims, strides, box)) return PREFILL_ERR_CUDA;
    }
    p.M = M;
    p.N = N;
    p.K = K;
    return pf::launch_qkv_gemm(tm_x, tm_w, p, tile_n, stream) == 0 ? PREFILL_OK : PREFILL_ERR_CUDA;
}

}  // namespace

extern "C" {

int qkv_projection(const prefill_bf16 *x, const prefill_bf16 *w, int tokens, int hidden, int n_head, int n_kv_head,
                   int head_dim, prefill_bf16 *q, prefill_bf16 *k, prefill_bf16 *v, int32_t *status_dev,
                   prefill_stream_t stream) {
    if (!x || !w || !q || !k || !v) return PREFILL_ERR_NULL;
    if (tokens < 0 || hidden < 0 || n_head < 1 || n_kv_head < 1 || head_dim < 1) return PREFILL_ERR_SHAPE;
    if (head_dim % 32 != 0 || hidden % 64 != 0 || hidden == 0) return PREFILL_ERR_UNSUPPORTED;
    const long long N = (long long)(n_head + 2 * n_kv_head) * head_dim;
    if (N % 256 != 0 || N > (1 << 30) || hidden > (1 << 30)) return PREFILL_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(w) || !aligned16(q) || !aligned16(k) || !aligned16(v)) return PREFILL_ERR_ALIGNMENT;
    if (tokens == 0) return PREFILL_OK;
    pf::QkvParams p;
    p.q = q;
    p.k = k;
    p.v = v;
    p.hq = n_head * head_dim;
    p.hkv = n_kv_head * head_dim;
    p.status = status_dev;
    return run_linear(x, w, tokens, hidden, (int)N, p, stream);
}

int attn_out_projection(const prefill_bf16 *o, const prefill_bf16 *w_o, int tokens, int n_head, int head_dim,
                        int hidden, prefill_bf16 *y, int32_t *status_dev, prefill_stream_t stream) {
    if (!o || !w_o || !y) return PREFILL_ERR_NULL;
    if (tokens < 0 || n_head < 1 || head_dim < 1 || hidden < 1) return PREFILL_ERR_SHAPE;
    const long long K = (long long)n_head * head_dim;
    if (K % 64 != 0 || hidden % 256 != 0 || K > (1 << 30) || hidden > (1 << 30)) return PREFILL_ERR_UNSUPPORTED;
    if (!aligned16(o) || !aligned16(w_o) || !aligned16(y)) return PREFILL_ERR_ALIGNMENT;
    if (tokens == 0) return PREFILL_OK;
    pf::QkvParams p;  // one output range: every column goes to y
    p.q = y;
    p.k = nullptr;
    p.v = nullptr;
    p.hq = hidden;
    p.hkv = 0;
    p.status = status_dev;
    return run_linear(o, w_o, tokens, (int)K, hidden, p, stream);
}

void prefill_test_inject_stall(int enable) { g_test_stall.store(enable ? 1 : 0); }

int prefill_test_exp2_fma2(const float *x, float *y, int n, prefill_stream_t stream) {
    if (n < 0) return PREFILL_ERR_SHAPE;
    if (n > 0 && (!x || !y)) return PREFILL_ERR_NULL;
    return pf::launch_exp2_fma2_probe(x, y, n, stream) == 0 ? PREFILL_OK : PREFILL_ERR_CUDA;
}

const char *prefill_status_string(int s) {
    switch (s) {
        case PREFILL_OK: return "ok";
        case PREFILL_ERR_NULL: return "a required pointer is NULL";
        case PREFILL_ERR_SHAPE: return "inconsistent sizes";
        case PREFILL_ERR_UNSUPPORTED: return "unsupported head_dim, block_size or scale";
        case PREFILL_ERR_BLOCK_TABLE: return "block table entry out of range or table too short";
        case PREFILL_ERR_CUDA: return "CUDA launch or driver failure";
        case PREFILL_ERR_TIMEOUT: return "device pipeline wait exceeded its limit";
        case PREFILL_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case PREFILL_ERR_SCRATCH_LIMIT:
            return "the call would need more split-KV scratch than the no-allocation entry point's static buffer holds";
        default: return "unknown status";
    }
}

int prefill_num_kv_blocks(int qb, int ctx, int n, int bm, int bn) {
    if (bm < 1 || bn < 1 || ctx < 0 || n < 0) return 0;
    return pf::num_kv_blocks(qb, ctx, n, bm, bn);
}

int prefill_kv_block_rule(int qb, int j, int ctx, int n, int bm, int bn, int32_t *col_limit, int32_t *key_begin) {
    return prefill_kv_block_rule_window(qb, j, ctx, n, bm, bn, 0, nullptr, col_limit, key_begin);
}

int prefill_first_kv_block(int qb, int ctx, int n, int bm, int bn, int window) {
    if (bm < 1 || bn < 1 || ctx < 0 || n < 0 || window < 0) return 0;
    return pf::first_kv_block(qb, ctx, n, bm, bn, window);
}

int prefill_kv_block_rule_window(int qb, int j, int ctx, int n, int bm, int bn, int window, int32_t *col_lo,
                                 int32_t *col_limit, int32_t *key_begin) {
    if (bm < 1 || bn < 1 || ctx < 0 || n < 0 || window < 0) return -1;
    if (j < prefill_first_kv_block(qb, ctx, n, bm, bn, window) || j >= prefill_num_kv_blocks(qb, ctx, n, bm, bn))
        return -1;
    const pf::KvBlock b = pf::kv_block(qb, j, ctx, n, bm, bn, window);
    if (key_begin) *key_begin = b.key_begin;
    for (int r = 0; r < bm; ++r) {
        if (col_limit) col_limit[r] = b.full ? bn : pf::col_limit(b, r, bn);
        if (col_lo) col_lo[r] = b.full ? 0 : pf::col_lo(b, r, bn);
    }
    return b.full ? 0 : 1;
}

}  // extern "C"
