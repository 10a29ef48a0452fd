// C ABI of the Titans neural long-term memory library: argument checks, dispatch
// to the kernels, tensor-map encoding and the device status word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <string>

#include "../../include/titans_mem.h"
#include "kernels.h"

struct titans_mem {
    titans_mem_config cfg;
    int device;
    unsigned* status;   // device status word
    float* ws;          // CUDA-core path workspace
    size_t ws_per_unit; // floats
};

namespace {

thread_local std::string g_err;

titans_status_t fail(titans_status_t s, const std::string& msg) {
    g_err = msg;
    return s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [units][T][64] bf16 viewed as a 3-D tensor {64, T, units}; box {64, chunk, 1}, 128-B swizzle,
// out-of-range rows read as zero.
bool encode_tokens(CUtensorMap* m, const void* base, long T, long units, int chunk) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {64, (cuuint64_t)T, (cuuint64_t)units};
    cuuint64_t strides[2] = {64 * 2, (cuuint64_t)T * 64 * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)chunk, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tc_eligible(const titans_mem_config& c, int chunk) {
    return c.mode == TITANS_BF16 && !(c.flags & TITANS_FLAG_CUDA_CORES) && c.d == 64 && c.d_hidden == 256 &&
           chunk >= 1 && chunk <= 64;
}

titans_status_t check_cfg(const titans_mem_config* c) {
    if (!c) return fail(TITANS_EINVAL, "config is NULL");
    if (c->B <= 0 || c->H <= 0) return fail(TITANS_EINVAL, "B and H must be positive");
    if ((long)c->B * c->H > (1L << 30)) return fail(TITANS_EINVAL, "too many units");
    if (c->d != 64 && c->d != 128) return fail(TITANS_EUNSUPPORTED, "d must be 64 or 128");
    if (c->d_hidden != 0 && c->d_hidden != 4 * c->d)
        return fail(TITANS_EUNSUPPORTED, "d_hidden must be 0 (linear memory) or 4*d");
    if (c->chunk < 1 || c->chunk > 128) return fail(TITANS_EUNSUPPORTED, "chunk must be in 1..128");
    if (c->mode != TITANS_BF16 && c->mode != TITANS_FP32) return fail(TITANS_EINVAL, "unknown mode");
    return TITANS_OK;
}

titans_status_t check_ptrs(const titans_mem* m, const void* k, const void* q, const void* v, const float* al,
                           const float* et, const float* th, const float* W1, const float* W2, const float* S1,
                           const float* S2, const void* y) {
    const void* req[] = {k, q, v, W1, S1, y};
    const char* names[] = {"k", "q", "v", "W1", "S1", "y"};
    for (int i = 0; i < 6; ++i) {
        if (!req[i]) return fail(TITANS_EINVAL, std::string(names[i]) + " is NULL");
        if (!aligned16(req[i])) return fail(TITANS_EINVAL, std::string(names[i]) + " is not 16-byte aligned");
    }
    const void* gates[] = {al, et, th};
    const char* gnames[] = {"alpha", "eta", "theta"};
    for (int i = 0; i < 3; ++i) {
        if (!gates[i]) return fail(TITANS_EINVAL, std::string(gnames[i]) + " is NULL");
        if (reinterpret_cast<uintptr_t>(gates[i]) & 3u)
            return fail(TITANS_EINVAL, std::string(gnames[i]) + " is not 4-byte aligned");
    }
    if (m->cfg.d_hidden) {
        if (!W2 || !S2) return fail(TITANS_EINVAL, "W2 and S2 are required for the MLP memory");
        if (!aligned16(W2) || !aligned16(S2)) return fail(TITANS_EINVAL, "W2/S2 not 16-byte aligned");
    }
    return TITANS_OK;
}

titans::ForwardArgs make_args(titans_mem* m, const void* k, const void* q, const void* v, const float* al,
                              const float* et, const float* th, long T, int chunk, float* W1, float* W2, float* S1,
                              float* S2, void* y) {
    titans::ForwardArgs a{};
    a.d = m->cfg.d;
    a.h = m->cfg.d_hidden;
    a.units = (long)m->cfg.B * m->cfg.H;
    a.T = T;
    a.chunk = chunk;
    a.bf16 = m->cfg.mode == TITANS_BF16;
    a.k = k;
    a.q = q;
    a.v = v;
    a.alpha = al;
    a.eta = et;
    a.theta = th;
    a.W1 = W1;
    a.W2 = W2;
    a.S1 = S1;
    a.S2 = S2;
    a.y = y;
    a.ws = m->ws;
    a.ws_per_unit = m->ws_per_unit;
    a.status = m->status;
    return a;
}

titans_status_t cuda_fail(cudaError_t e, const char* what) {
    return fail(TITANS_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

}  // namespace

namespace titans {
// Lets the library's other entry points report through titans_last_error_string().
void set_last_error(const std::string& msg) { g_err = msg; }
}  // namespace titans

extern "C" {

int titans_mem_version(void) { return 100; }

const char* titans_last_error_string(void) { return g_err.c_str(); }

titans_status_t titans_mem_init(const titans_mem_config* cfg, titans_mem_t* out) {
    if (!out) return fail(TITANS_EINVAL, "out is NULL");
    *out = nullptr;
    titans_status_t s = check_cfg(cfg);
    if (s != TITANS_OK) return s;
    titans_mem* m = new titans_mem();
    m->cfg = *cfg;
    cudaError_t e = cudaGetDevice(&m->device);
    if (e != cudaSuccess) {
        delete m;
        return cuda_fail(e, "cudaGetDevice");
    }
    e = cudaMalloc(&m->status, sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemset(m->status, 0, sizeof(unsigned));
    if (e != cudaSuccess) {
        delete m;
        return cuda_fail(e, "allocating the status word");
    }
    m->ws_per_unit = titans::cuda_cores_ws_floats(cfg->d, cfg->d_hidden, cfg->chunk);
    m->ws_per_unit = (m->ws_per_unit + 63) & ~size_t(63);
    e = cudaMalloc(&m->ws, m->ws_per_unit * sizeof(float) * (size_t)cfg->B * cfg->H);
    if (e != cudaSuccess) {
        cudaFree(m->status);
        delete m;
        return cuda_fail(e, "allocating the workspace");
    }
    *out = m;
    return TITANS_OK;
}

titans_status_t titans_mem_destroy(titans_mem_t m) {
    if (!m) return fail(TITANS_EINVAL, "handle is NULL");
    cudaFree(m->ws);
    cudaFree(m->status);
    delete m;
    return TITANS_OK;
}

int titans_mem_path(titans_mem_t m, int chunk, int step) {
    if (!m) return -1;
    if (step) return m->cfg.d_hidden ? TITANS_PATH_STEP_CLUSTER : TITANS_PATH_CUDA_CORES;
    if (chunk < 1 || chunk > m->cfg.chunk) return -1;
    return tc_eligible(m->cfg, chunk) ? TITANS_PATH_TC_MLP64 : TITANS_PATH_CUDA_CORES;
}

titans_status_t titans_mem_forward(titans_mem_t m, const void* k, const void* q, const void* v, const float* alpha,
                                   const float* eta, const float* theta, long T, int chunk, float* W1, float* W2,
                                   float* S1, float* S2, void* y, void* stream) {
    if (!m) return fail(TITANS_EINVAL, "handle is NULL");
    titans_status_t s = check_ptrs(m, k, q, v, alpha, eta, theta, W1, W2, S1, S2, y);
    if (s != TITANS_OK) return s;
    if (T < 1) return fail(TITANS_EINVAL, "T must be >= 1");
    if (T * (long)m->cfg.d >= (1L << 31)) return fail(TITANS_EUNSUPPORTED, "T * d must be below 2^31");
    if (chunk < 1 || chunk > m->cfg.chunk)
        return fail(TITANS_EUNSUPPORTED, "chunk must be in 1..config.chunk");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    titans::ForwardArgs a = make_args(m, k, q, v, alpha, eta, theta, T, chunk, W1, W2, S1, S2, y);
    cudaError_t e;
    if (tc_eligible(m->cfg, chunk)) {
        if (T >= (1L << 31) || a.units >= (1L << 31)) return fail(TITANS_EUNSUPPORTED, "T or units too large");
        CUtensorMap tk, tq, tv;
        if (!encode_tokens(&tk, k, T, a.units, chunk) || !encode_tokens(&tq, q, T, a.units, chunk) ||
            !encode_tokens(&tv, v, T, a.units, chunk))
            return fail(TITANS_ECUDA, "cuTensorMapEncodeTiled failed");
        e = titans::launch_chunk_tc_mlp64(a, tk, tq, tv, st);
    } else {
        e = titans::launch_chunk_cuda_cores(a, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return TITANS_OK;
}

titans_status_t titans_mem_step(titans_mem_t m, const void* k, const void* q, const void* v, const float* alpha,
                                const float* eta, const float* theta, float* W1, float* W2, float* S1, float* S2,
                                void* y, void* stream) {
    if (!m) return fail(TITANS_EINVAL, "handle is NULL");
    titans_status_t s = check_ptrs(m, k, q, v, alpha, eta, theta, W1, W2, S1, S2, y);
    if (s != TITANS_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    titans::ForwardArgs a = make_args(m, k, q, v, alpha, eta, theta, 1, 1, W1, W2, S1, S2, y);
    cudaError_t e = m->cfg.d_hidden ? titans::launch_step_cluster(a, st) : titans::launch_chunk_cuda_cores(a, st);
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return TITANS_OK;
}

titans_status_t titans_mem_sync_status(titans_mem_t m, void* stream) {
    if (!m) return fail(TITANS_EINVAL, "handle is NULL");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned h = 0;
    e = cudaMemcpy(&h, m->status, sizeof(unsigned), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(m->status, 0, sizeof(unsigned));
    if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
    if (h) {
        char buf[128];
        snprintf(buf, sizeof buf, "device status 0x%x (1: TMA wait timed out, 2: MMA wait timed out)", h);
        return fail(TITANS_EDEVICE, buf);
    }
    return TITANS_OK;
}

}  // extern "C"
