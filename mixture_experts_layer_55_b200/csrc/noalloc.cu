// noalloc.cu -- moe_dispatch_noalloc: the dispatch with its scratch memory in
// a static device array instead of a caller-allocated workspace.
//
// For callers that are handed only their input and output buffers and may not
// allocate device memory themselves (for example a plugin enqueued by a host
// inference framework, or a C program with a fixed memory budget): they have
// no workspace to pass, and cudaMalloc is not open to them because it can
// synchronise the device and falls outside the memory they were budgeted.
//
// The scratch (device status word, per-chunk expert counts and rank bases)
// lives in g_noalloc_scratch, kNoallocScratchBytes = 256 KiB, which every GPU
// that loads the library holds until the process exits.  In host code the
// array's name is only a host-side stand-in, so every call looks up its device
// address on the current device with cudaGetSymbolAddress.  The lookup is a
// table read once the library's device code is loaded on that device (the
// first call there loads it); it is repeated on every call rather than cached
// so that a cudaDeviceReset, after which the array may sit at a new address,
// leaves no stale pointer behind.
#include "internal.h"

namespace moe {

constexpr size_t kNoallocScratchBytes = 256 * 1024;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of the static scratch on the current device.
static cudaError_t noalloc_scratch(char** out)
{
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    *out = static_cast<char*>(p);
    return cudaSuccess;
}

// The dispatch kernels' scratch regions packed into the static array.
static WsLayout noalloc_layout(const moe_config& c)
{
    const int64_t nch = dispatch_chunks(c);
    WsLayout L{};
    L.status = 0;
    L.d_cnt = align_up(64 * sizeof(int));
    L.d_base = L.d_cnt + align_up((size_t)nch * c.E * sizeof(int32_t));
    L.total = L.d_base + align_up((size_t)nch * c.E * sizeof(int32_t));
    return L;
}

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_dispatch_noalloc(const moe_config* cfg, const void* x,
                                           const int32_t* topk_ids, int32_t* counts,
                                           int32_t* kept, int32_t* offsets, int32_t* perm,
                                           int32_t* row_of, void* x_perm, void* stream)
{
    moe_status st = moe_check_config(cfg);
    if (st != MOE_OK) return st;
    if (!topk_ids || !counts || !kept || !offsets || !perm || !row_of) return MOE_ERR_ARG;
    if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_ARG;
    if (x && (((uintptr_t)x & 15u) != 0 || ((uintptr_t)x_perm & 15u) != 0)) return MOE_ERR_ALIGN;
    const WsLayout L = noalloc_layout(*cfg);
    if (L.total > kNoallocScratchBytes) return MOE_ERR_WORKSPACE;  // beyond the static array
    char* scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) return cuda_status(e);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the status word collects flags with atomic OR: it must start at zero
    e = cudaMemsetAsync(scratch + L.status, 0, 64 * sizeof(int), s);
    if (e == cudaSuccess) {
        int64_t C = 0;
        moe_capacity(cfg, &C);
        e = launch_dispatch_index(*cfg, C, topk_ids, counts, kept, offsets, perm, row_of, scratch,
                                  L, s);
    }
    if (e == cudaSuccess && x) {
        int64_t rows = 0;
        moe_max_rows(cfg, &rows);
        e = launch_gather(*cfg, x, row_of, x_perm, rows, reinterpret_cast<int*>(scratch + L.status),
                          s);
    }
    return cuda_status(e);
}

extern "C" moe_status moe_dispatch_noalloc_status(void* stream, int32_t* flags)
{
    if (flags == nullptr) return MOE_ERR_ARG;
    char* scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) return cuda_status(e);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t word = 0;  // word 0 of the status region (offset 0 of the layout)
    e = cudaMemcpyAsync(&word, scratch, sizeof word, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e);
    *flags = word;
    if (word & MOE_DEVFLAG_TIMEOUT) return MOE_ERR_DEVICE_TIMEOUT;
    if (word & MOE_DEVFLAG_BOUNDS) return MOE_ERR_DEVICE_BOUNDS;
    return MOE_OK;
}
