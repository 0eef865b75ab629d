// decode_paged_noalloc.cu -- paged decode for callers that cannot allocate
// device memory.
//
// paged_attn_decode needs a caller-provided workspace (split-KV partial
// outputs, their logsumexps, the per-sequence split offsets and a work
// counter).  Some callers have no way to provide one: code that runs where
// cudaMalloc is not allowed or not wanted (inside a custom allocator or a
// memory-pool callback, in a process whose allocations are fixed up front,
// or a plain C host program with no tensor framework to borrow memory from).
// This entry point uses a fixed scratch array compiled into the library
// instead, so it calls no allocator at all.
//
// Costs and rules of the static scratch:
//   * kNoAllocScratchBytes of device memory are reserved on every GPU that
//     loads this library's device code, for the life of the process.
//   * Sizes whose workspace would exceed it are rejected (ATTN_EUNSUPPORTED)
//     before anything is launched.
//   * All calls on a device share the one array.  Two calls whose kernels
//     overlap on the GPU (different streams without ordering between them)
//     race on it and give wrong results; calls on one stream are ordered.
//   * The array keeps whatever the previous call left there.  Three areas of
//     it must start at zero: the work counter, the per-(sequence, head)
//     completion counts (done_cnt) and the per-sequence bad-block marks
//     (seq_bad).  decode_plan_kernel, the first kernel of every call,
//     clears all three; every other byte is written before it is read.  A
//     change that adds another counter must clear it there too.
//   * The scratch used is the current device's: the tensors' device must be
//     current when the function is called (the address of another device's
//     array would be read as garbage on this one).
//   * The scratch address is looked up once per device, on the first call
//     made while that device is current.  Make that first call before any
//     stream capture begins, since the lookup is a runtime call.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/attn.h"
#include "launch.h"

namespace {

constexpr size_t kNoAllocScratchBytes = ATTN_NOALLOC_SCRATCH_BYTES;
static_assert(kNoAllocScratchBytes % 256 == 0, "scratch size must keep 256-byte alignment");

// The scratch itself.  In host code this name is only a handle for the
// runtime; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_decode_scratch on the current device (looked up once).
attn_status scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ECUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return ATTN_ECUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return ATTN_OK;
}

}  // namespace

extern "C" ATTN_API attn_status paged_attn_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                                          const int32_t *block_table, const int32_t *seq_lens,
                                                          int block_size, void *O, float *LSE, int num_seqs, int H,
                                                          int d, int num_blocks, int max_blocks_per_seq,
                                                          float scale, attn_dtype dt, int32_t *err_flag,
                                                          attn_stream_t stream) {
    // the sizes are checked by paged_attn_decode itself; here only the fit
    const size_t need = paged_attn_decode_workspace_size(num_seqs, H, d, max_blocks_per_seq, block_size);
    if (need > kNoAllocScratchBytes) return ATTN_EUNSUPPORTED;
    if (num_seqs == 0) return paged_attn_decode(q, k_cache, v_cache, block_table, seq_lens, block_size, O, LSE,
                                                num_seqs, H, d, num_blocks, max_blocks_per_seq, scale, dt, nullptr, 0,
                                                err_flag, stream);
    void *scratch = nullptr;
    const attn_status st = scratch_address(&scratch);
    if (st != ATTN_OK) return st;
    return paged_attn_decode(q, k_cache, v_cache, block_table, seq_lens, block_size, O, LSE, num_seqs, H, d,
                             num_blocks, max_blocks_per_seq, scale, dt, scratch, kNoAllocScratchBytes, err_flag,
                             stream);
}
