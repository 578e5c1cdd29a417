// noalloc.cu -- prefill_attn_chunked_noalloc: chunked prefill for callers that
// cannot let the library allocate device memory.
//
// prefill_attn_chunked may need a split-KV workspace, which the library obtains
// with cudaMalloc on the first call that splits.  Some callers cannot allow
// that: engines that own all device memory through their own pool and forbid
// allocations behind its back, and hosts whose memory budget is fixed at
// start-up.  This entry point runs the same kernels with the split partials in
// a fixed, file-scope device array instead, and never calls cudaMalloc,
// cudaFree or any allocating routine.  A call whose split partials would not
// fit the array runs with fewer splits (down to none).
//
// The array is kScratchBytes (32 MiB) on every GPU that loads this library,
// held until the process exits.  Every call shares it and it keeps the last
// call's contents; nothing in it has to start at zero (each call writes every
// partial it later reads).  Calls whose work overlaps on the GPU -- on two
// streams, or on the same device from two threads without ordering -- race on
// the array and must be serialised by the caller.
#include <cuda_runtime.h>

#include <cstdint>
#include <map>
#include <mutex>

#include "../../include/prefill.h"
#include "params.h"

namespace {

constexpr size_t kScratchBytes = 32u << 20;

static __device__ __align__(256) unsigned char g_split_scratch[kScratchBytes];

std::mutex g_mu;
std::map<int, void *> g_scratch_addr;  // device -> address of g_split_scratch on it

// The array's device address on the current device, looked up once per device
// (the first call on a device does this set-up).  In host code the symbol
// names a host-side stand-in, never a device address, so only this address is
// passed to the kernels.
void *scratch_address(cudaError_t *err) {
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_scratch_addr.find(dev);
    if (it != g_scratch_addr.end()) return it->second;
    void *ptr = nullptr;
    *err = cudaGetSymbolAddress(&ptr, g_split_scratch);
    if (*err != cudaSuccess || ptr == nullptr) return nullptr;
    g_scratch_addr[dev] = ptr;
    return ptr;
}

}  // namespace

extern "C" {

int prefill_attn_chunked_noalloc(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v, int total_q,
                                 const int32_t *cu_seqlens_q, const int32_t *context_lens, int num_seqs,
                                 int max_q_len, int max_context_len, int n_head, int n_kv_head, int head_dim,
                                 float scale, prefill_bf16 *out, prefill_bf16 *kv_cache, int num_blocks,
                                 const int32_t *block_table, int max_blocks_per_seq, int block_size,
                                 int32_t *status_dev, prefill_stream_t stream) {
    cudaError_t err = cudaSuccess;
    void *scratch = scratch_address(&err);
    if (!scratch) {
        cudaGetLastError();
        return PREFILL_ERR_CUDA;
    }
    return pf::run_prefill(q, k, v, total_q, cu_seqlens_q, context_lens, true, num_seqs, max_q_len, max_context_len,
                           n_head, n_kv_head, head_dim, scale, out, kv_cache, num_blocks, block_table,
                           max_blocks_per_seq, block_size, status_dev, stream, scratch, kScratchBytes);
}

size_t prefill_noalloc_scratch_bytes(void) { return kScratchBytes; }

}  // extern "C"
