// titans_mem_forward_noalloc: the chunk-wise forward for callers that cannot allocate
// device memory.
//
// Who needs it: code that runs where cudaMalloc is off limits or unsafe -- inside a CUDA
// graph being captured by someone else's framework, under an allocator that owns all
// device memory (a serving engine's memory pool), in a real-time path that must not
// synchronize the device (cudaMalloc may), or in a plug-in that must not leave
// allocations behind. titans_mem_init cannot serve them: it allocates the handle's status
// word and workspace.
//
// What it does: runs the CUDA-core (fp32 arithmetic) chunk kernel, the same kernel that
// titans_mem_forward runs with TITANS_FLAG_CUDA_CORES, with its per-unit scratch taken
// from a fixed array compiled into the library instead of from a handle. The array is
// kNoallocScratchBytes (16 MiB) of device memory that every GPU which loads the library
// holds until the process exits.
//
// Rules for callers:
//  - The first call on a device looks up the array's device address there
//    (cudaGetSymbolAddress, with that device current) and loads the kernel's code for both
//    input dtypes (cudaFuncGetAttributes), so that no later call, in either mode, makes the
//    runtime load code. Make that first call before any stream capture that should contain
//    a later call.
//  - All calls share the one array: calls whose kernels overlap on a GPU (different
//    streams, or host threads) race on it and corrupt each other's results. Serialize them.
//  - The array keeps the last call's contents; the kernel writes every scratch element of
//    a chunk before reading it, so nothing needs clearing between calls.
//  - Calls needing more scratch than the array holds are rejected (TITANS_EUNSUPPORTED):
//    4*chunk*h + chunk*d floats per unit for the MLP memory, chunk*d for the linear one,
//    each rounded up to 64 floats, times B*H units.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <string>

#include "../../include/titans_mem.h"
#include "kernels.h"

namespace titans {

void set_last_error(const std::string& msg);  // api.cu

constexpr size_t kNoallocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) float g_noalloc_scratch[kNoallocScratchBytes / sizeof(float)];

namespace {

titans_status_t fail(titans_status_t s, const std::string& m) {
    set_last_error(m);
    return s;
}

// Device address of g_noalloc_scratch for the current device. In host code the array's
// name is a host-side stand-in, not a device address, so it is looked up once per device
// (with that device current) and cached. The same first call loads the CUDA-core kernel's
// fp32- and bf16-input instantiations on that device.
constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_ptr[kMaxDevices] = {};

cudaError_t scratch_for_current_device(float** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        e = preload_chunk_cuda_cores();
        if (e != cudaSuccess) return e;
        g_ptr[dev] = static_cast<float*>(p);
    }
    *out = g_ptr[dev];
    return cudaSuccess;
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace titans

extern "C" titans_status_t titans_mem_forward_noalloc(const titans_mem_config* cfg, const void* k, const void* q,
                                                      const void* v, const float* alpha, const float* eta,
                                                      const float* theta, long T, int chunk, float* W1, float* W2,
                                                      float* S1, float* S2, void* y, void* stream) {
    using namespace titans;
    if (!cfg) return fail(TITANS_EINVAL, "config is NULL");
    if (cfg->B <= 0 || cfg->H <= 0) return fail(TITANS_EINVAL, "B and H must be positive");
    if ((long)cfg->B * cfg->H > (1L << 30)) return fail(TITANS_EINVAL, "too many units");
    if (cfg->d != 64 && cfg->d != 128) return fail(TITANS_EUNSUPPORTED, "d must be 64 or 128");
    if (cfg->d_hidden != 0 && cfg->d_hidden != 4 * cfg->d)
        return fail(TITANS_EUNSUPPORTED, "d_hidden must be 0 (linear memory) or 4*d");
    if (cfg->mode != TITANS_BF16 && cfg->mode != TITANS_FP32) return fail(TITANS_EINVAL, "unknown mode");
    if (chunk < 1 || chunk > 128) return fail(TITANS_EUNSUPPORTED, "chunk must be in 1..128");
    if (T < 1) return fail(TITANS_EINVAL, "T must be >= 1");
    if (T * (long)cfg->d >= (1L << 31)) return fail(TITANS_EUNSUPPORTED, "T * d must be below 2^31");
    const void* req[] = {k, q, v, W1, S1, y};
    for (const void* p : req)
        if (!p || !a16(p)) return fail(TITANS_EINVAL, "k, q, v, W1, S1, y must be non-NULL and 16-byte aligned");
    const void* gates[] = {alpha, eta, theta};
    for (const void* p : gates)
        if (!p || (reinterpret_cast<uintptr_t>(p) & 3u))
            return fail(TITANS_EINVAL, "alpha, eta, theta must be non-NULL and 4-byte aligned");
    if (cfg->d_hidden && (!W2 || !S2 || !a16(W2) || !a16(S2)))
        return fail(TITANS_EINVAL, "W2 and S2 must be non-NULL and 16-byte aligned for the MLP memory");

    const long units = (long)cfg->B * cfg->H;
    size_t per_unit = cuda_cores_ws_floats(cfg->d, cfg->d_hidden, chunk);
    per_unit = (per_unit + 63) & ~size_t(63);
    // units <= 2^30 and per_unit < 2^20 floats, so the product cannot wrap.
    const size_t need = per_unit * sizeof(float) * (size_t)units;
    if (need > kNoallocScratchBytes)
        return fail(TITANS_EUNSUPPORTED, "scratch of " + std::to_string(need) + " bytes (B*H units x chunk) exceeds " +
                                             "the fixed " + std::to_string(kNoallocScratchBytes) +
                                             "-byte array of titans_mem_forward_noalloc");
    float* scratch = nullptr;
    cudaError_t e = scratch_for_current_device(&scratch);
    if (e != cudaSuccess) return fail(TITANS_ECUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));

    ForwardArgs a{};
    a.d = cfg->d;
    a.h = cfg->d_hidden;
    a.units = units;
    a.T = T;
    a.chunk = chunk;
    a.bf16 = cfg->mode == TITANS_BF16;
    a.k = k;
    a.q = q;
    a.v = v;
    a.alpha = alpha;
    a.eta = eta;
    a.theta = theta;
    a.gate_ld = T;
    a.W1 = W1;
    a.W2 = W2;
    a.S1 = S1;
    a.S2 = S2;
    a.y = y;
    a.ws = scratch;
    a.ws_per_unit = per_unit;
    a.status = nullptr;  // the CUDA-core kernel has no waits to time out
    e = launch_chunk_cuda_cores(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(TITANS_ECUDA, std::string("kernel launch: ") + cudaGetErrorString(e));
    return TITANS_OK;
}
