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
// host-side stand-in), so the device address is looked up with
// cudaGetSymbolAddress, with the device current, on the first call made on
// it, and looked up again if the device's context has changed since (a
// cudaDeviceReset, or another context made current); make that first call
// before any stream capture.  Calls share the array and it keeps the last
// call's contents; the decode kernels write every partial they later read, so
// nothing has to start at zero.  Calls that may overlap on the GPU (other
// streams, other host threads) race on the array: the caller must order them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/fa.h"
#include "fa_internal.h"

namespace fa {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;

// Cached address per device, valid for the context whose unique ID it
// records (IDs are never reused within a process, unlike context handles).
struct ScratchEntry {
    unsigned long long ctx_id;
    void *ptr;
};
ScratchEntry g_scratch[kMaxDevices];
std::mutex g_scratch_mutex;

using PfnCtxGetCurrent = CUresult (*)(CUcontext *);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long *);

// ID of the calling thread's current context; false if none is current or
// the driver entry points are unavailable.
bool current_context_id(unsigned long long *id) {
    static std::once_flag once;
    static PfnCtxGetCurrent get_current = nullptr;
    static PfnCtxGetId get_id = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PfnCtxGetCurrent>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PfnCtxGetId>(p);
    });
    if (!get_current || !get_id) return false;
    CUcontext c = nullptr;
    if (get_current(&c) != CUDA_SUCCESS || !c) return false;
    return get_id(c, id) == CUDA_SUCCESS;
}

// Device address of the scratch array on the current device.  Returns nullptr
// on failure.
void *noalloc_scratch_address() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    unsigned long long id = 0;
    if (current_context_id(&id)) {
        std::lock_guard<std::mutex> lock(g_scratch_mutex);
        if (g_scratch[dev].ptr && g_scratch[dev].ctx_id == id) return g_scratch[dev].ptr;
    }
    // Set-up (first call on this device, or its context changed): the lookup
    // also makes the runtime's context current when none was.
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) return nullptr;
    if (current_context_id(&id)) {
        std::lock_guard<std::mutex> lock(g_scratch_mutex);
        g_scratch[dev] = ScratchEntry{id, addr};
    }
    return addr;
}

}  // namespace

}  // namespace fa

extern "C" {

int fa_decode_paged_noalloc(const void *q, const void *k_cache, const void *v_cache,
                            const int *block_table, const int *seq_lens, void *o, float *lse,
                            int num_seqs, int num_pages, int Hq, int Hkv, int d, int page_size,
                            int max_pages_per_seq, float scale, void *stream) {
    // Every argument check of fa_decode_paged runs first, with no workspace:
    // it calls no CUDA function and returns FA_ERR_WORKSPACE only once all
    // other arguments are valid (FA_OK for an empty batch).
    int rc = fa_decode_paged(q, k_cache, v_cache, block_table, seq_lens, o, lse, num_seqs,
                             num_pages, Hq, Hkv, d, page_size, max_pages_per_seq, scale,
                             nullptr, 0, stream);
    if (rc != FA_ERR_WORKSPACE) return rc;
    // Then the size: a request whose scratch would not fit in the fixed
    // array is refused before any CUDA call.
    const size_t need = fa_decode_workspace_bytes(num_seqs, Hq, d, page_size, max_pages_per_seq);
    if (need > fa::kNoAllocScratchBytes) return FA_ERR_WORKSPACE;
    void *scratch = fa::noalloc_scratch_address();
    if (!scratch) return FA_ERR_CUDA;
    return fa_decode_paged(q, k_cache, v_cache, block_table, seq_lens, o, lse, num_seqs,
                           num_pages, Hq, Hkv, d, page_size, max_pages_per_seq, scale, scratch,
                           fa::kNoAllocScratchBytes, stream);
}

}  // extern "C"
