// decode_noalloc.cu -- fa_decode_paged_noalloc: paged decode for callers that
// cannot allocate device memory.
//
// fa_decode_paged needs a caller-provided workspace for its split-KV partial
// results.  Some callers cannot provide one: code that runs inside a host
// framework whose memory pool owns the device and forbids raw cudaMalloc,
// latency-critical serving paths where cudaMalloc's implicit device
// synchronisation is not allowed, or embedded callers with a fixed memory
// budget decided at load time.  For them this entry point takes its scratch
// from a fixed array in the library's own device memory instead.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes
// (32 MiB).  Every GPU that loads the library holds it until the process
// exits.  Host code cannot use the array's name as a device address (it is a
// host-side stand-in), so the device address is looked up once per device
// with cudaGetSymbolAddress, with that device current, on the first call made
// on it; make that first call before any stream capture.  Calls share the
// array and it keeps the last call's contents; the decode kernels write every
// partial they later read, so nothing has to start at zero.  Calls that may
// overlap on the GPU (other streams, other host threads) race on the array:
// the caller must order them.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "../../include/fa.h"
#include "fa_internal.h"

namespace fa {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device (set-up on the
// first call per device).  Returns nullptr on failure.
void *noalloc_scratch_address() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void *p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (p) return p;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (p) return p;
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) return nullptr;
    g_scratch_ptr[dev].store(addr, std::memory_order_release);
    return addr;
}

}  // namespace

}  // namespace fa

extern "C" {

int fa_decode_paged_noalloc(const void *q, const void *k_cache, const void *v_cache,
                            const int *block_table, const int *seq_lens, void *o, float *lse,
                            int num_seqs, int num_pages, int Hq, int Hkv, int d, int page_size,
                            int max_pages_per_seq, float scale, void *stream) {
    // Sizes are checked before any CUDA call: a request whose scratch would
    // not fit in the fixed array is refused with FA_ERR_WORKSPACE.
    if (num_seqs > 0 && max_pages_per_seq > 0) {
        const size_t need =
            fa_decode_workspace_bytes(num_seqs, Hq, d, page_size, max_pages_per_seq);
        if (need > fa::kNoAllocScratchBytes) return FA_ERR_WORKSPACE;
    }
    if (num_seqs == 0) {
        // Same argument checks as fa_decode_paged, without touching the device.
        return fa_decode_paged(q, k_cache, v_cache, block_table, seq_lens, o, lse, num_seqs,
                               num_pages, Hq, Hkv, d, page_size, max_pages_per_seq, scale,
                               nullptr, 0, stream);
    }
    void *scratch = fa::noalloc_scratch_address();
    if (!scratch) return FA_ERR_CUDA;
    return fa_decode_paged(q, k_cache, v_cache, block_table, seq_lens, o, lse, num_seqs,
                           num_pages, Hq, Hkv, d, page_size, max_pages_per_seq, scale, scratch,
                           fa::kNoAllocScratchBytes, stream);
}

}  // extern "C"
