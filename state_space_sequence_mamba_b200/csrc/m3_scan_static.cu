// m3_scan_fwd_noalloc: the prefill scan for callers that cannot give the library a workspace
// buffer.
//
// Some callers cannot allocate device memory at the point where they run the scan: a serving
// runtime that plans all of its device memory up front and forbids allocation while it serves,
// code that runs inside a step whose memory has been fixed in advance, or an embedding that
// simply has no allocator to offer. For them this entry point takes its scratch (the status
// header, the per-token RMS scales of B and C and, room permitting, the segment end states of
// the sequence-parallel form) from one array of fixed size that is part of the library itself,
// so the call needs nothing beyond its inputs and outputs. Few long sequences then run in as
// many segments as the array holds the end states of, down to one.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds its
// own copy of it until the process exits. Host code cannot use the variable's name as a
// device address, so the first call on each device looks the address up with
// cudaGetSymbolAddress while that device is current, and every later call on that device
// reuses the cached address.
#include <mutex>

#include "m3_internal.h"

namespace m3 {

constexpr size_t kStaticScratchBytes = size_t(1) << 20;  // 1 MiB

// The scratch itself: one per device that loads the library, alive until the process exits.
static __device__ __align__(256) unsigned char g_scan_scratch[kStaticScratchBytes];

namespace {

constexpr size_t kStatusBytes = 256;                       // header that must start at zero
constexpr int kMaxDevices = 64;

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

m3_status static_fail(m3_status s, const char* msg) { return set_error(s, msg); }

}  // namespace
}  // namespace m3

using namespace m3;

extern "C" {

M3_API m3_status m3_scan_fwd_noalloc(const m3_dims* dims, const m3_inputs* in,
                                     const m3_state* init, const m3_state* final_state,
                                     void* y, void* stream) {
    const size_t need = scan_workspace_min_bytes(dims);
    if (need == 0) {
        // invalid or unsupported dims: let the regular entry point say which, with no launch
        return m3_scan_fwd(dims, in, init, final_state, y, nullptr, 0, stream);
    }
    if (need > kStaticScratchBytes)
        return static_fail(M3_ERR_UNSUPPORTED,
                           "m3_scan_fwd_noalloc: these dims need more scratch than the "
                           "library's fixed 1 MiB (with BC normalisation on, batch * "
                           "ceil(seqlen / chunk) * chunk * ngroups * rank must be <= 131040); "
                           "use m3_scan_fwd");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return static_fail(M3_ERR_CUDA, "m3_scan_fwd_noalloc: no usable current device");
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        if (!g_scratch_addr[dev]) {
            void* p = nullptr;
            const cudaError_t e = cudaGetSymbolAddress(&p, g_scan_scratch);
            if (e != cudaSuccess || !p)
                return static_fail(M3_ERR_CUDA,
                                   "m3_scan_fwd_noalloc: cudaGetSymbolAddress of the scratch "
                                   "array failed");
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }
    // The array keeps whatever the previous call left; the status header must read zero.
    if (cudaMemsetAsync(scratch, 0, kStatusBytes, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return static_fail(M3_ERR_CUDA, "m3_scan_fwd_noalloc: clearing the status header failed");
    return scan_fwd_with(dims, in, init, final_state, y, scratch, kStaticScratchBytes, need, stream);
}

}  // extern "C"
