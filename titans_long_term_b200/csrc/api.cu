// C ABI of the Titans neural long-term memory library: argument checks, dispatch
// to the kernels, tensor-map encoding and the device status word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <algorithm>
#include <string>
#include <vector>

#include "../../include/titans_mem.h"
#include "kernels.h"

struct titans_mem {
    titans_mem_config cfg;
    int layers = 2;     // memory depth; titans_mem_init_deep sets it
    int nseg_max = 1;   // segments per unit of the linear memory's cross-chunk scan
    int device;
    unsigned* status;   // device status word, then the phased kernel's two grid-barrier words
    float* ws;          // CUDA-core path workspace
    size_t ws_per_unit; // floats
    // titans_mem_forward_host: copy streams and events, created on first use.
    cudaStream_t s_in = nullptr, s_out = nullptr;
    std::vector<cudaEvent_t> ev;  // [0] start, [1] done, then (copied in, computed) per segment
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

bool deep_tc_eligible(const titans_mem_config& c, int layers, int chunk) {
    return c.mode == TITANS_BF16 && !(c.flags & TITANS_FLAG_CUDA_CORES) &&
           titans::tc_deep_supported(c.d, c.d_hidden, layers, chunk);
}

bool backward_tc_eligible(const titans_mem_config& c, int chunk) {
    return c.mode == TITANS_BF16 && !(c.flags & TITANS_FLAG_CUDA_CORES) && c.d_hidden != 0 &&
           titans::mlp_backward_tc_supported(c.d, c.d_hidden, chunk);
}

bool phased_eligible(const titans_mem_config& c, int chunk) {
    return c.mode == TITANS_BF16 && !(c.flags & TITANS_FLAG_CUDA_CORES) &&
           titans::tc_phased_supported(c.d, c.d_hidden, chunk);
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
    a.chunk_gates = (m->cfg.flags & TITANS_FLAG_CHUNK_GATES) != 0;
    a.gate_ld = a.chunk_gates ? (T + chunk - 1) / chunk : T;
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

// Elements in one unit's gate row: T per-token gates, or one per chunk with TITANS_FLAG_CHUNK_GATES.
long gate_row(const titans_mem* m, long T, int chunk) {
    return (m && (m->cfg.flags & TITANS_FLAG_CHUNK_GATES) && chunk > 0) ? (T + chunk - 1) / chunk : T;
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

titans_status_t titans_silu_routes(const float* h, float* silu_fma, float* silu_mufu, long n, void* stream) {
    if (n < 0) return fail(TITANS_EINVAL, "titans_silu_routes: n < 0");
    if (n > 0 && (!h || !silu_fma || !silu_mufu)) return fail(TITANS_EINVAL, "titans_silu_routes: NULL pointer");
    const cudaError_t e = titans::launch_silu_routes(h, silu_fma, silu_mufu, n, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail(TITANS_ECUDA, std::string("titans_silu_routes: ") + cudaGetErrorString(e));
    return TITANS_OK;
}

const char* titans_last_error_string(void) { return g_err.c_str(); }

}  // extern "C"

namespace {
titans_status_t init_impl(const titans_mem_config* cfg, int layers, titans_mem_t* out) {
    if (!out) return fail(TITANS_EINVAL, "out is NULL");
    *out = nullptr;
    titans_status_t s = check_cfg(cfg);
    if (s != TITANS_OK) return s;
    if (layers != 2 && (layers < 2 || layers > 8)) return fail(TITANS_EUNSUPPORTED, "layers must be in 2..8");
    if (layers > 2 && cfg->d_hidden == 0) return fail(TITANS_EINVAL, "a deep memory needs d_hidden > 0");
    titans_mem* m = new titans_mem();
    m->cfg = *cfg;
    m->layers = layers;
    cudaError_t e = cudaGetDevice(&m->device);
    if (e != cudaSuccess) {
        delete m;
        return cuda_fail(e, "cudaGetDevice");
    }
    e = cudaMalloc(&m->status, 4 * sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemset(m->status, 0, 4 * sizeof(unsigned));
    if (e != cudaSuccess) {
        delete m;
        return cuda_fail(e, "allocating the status word");
    }
    m->ws_per_unit = titans::cuda_cores_ws_floats(cfg->d, cfg->d_hidden, cfg->chunk);
    if (cfg->d_hidden)
        m->ws_per_unit = std::max(m->ws_per_unit, titans::deep_ws_floats(cfg->d, cfg->d_hidden, layers, cfg->chunk));
    if (layers > 2 && deep_tc_eligible(*cfg, layers, cfg->chunk))
        m->ws_per_unit = std::max(m->ws_per_unit,
                                  (titans::tc_deep_ws_bytes_per_unit(cfg->d, cfg->d_hidden, layers) + 3) / sizeof(float));
    if (phased_eligible(*cfg, cfg->chunk))
        m->ws_per_unit = std::max(m->ws_per_unit, titans::tc_phased_ws_bytes_per_unit() / sizeof(float));
    if (cfg->d_hidden == 0 && (cfg->flags & TITANS_FLAG_CHUNK_SCAN)) {
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, m->device);
        if (e != cudaSuccess) {
            cudaFree(m->status);
            delete m;
            return cuda_fail(e, "querying the SM count");
        }
        // Enough segments to give every SM a CTA, at most 4096 per unit.
        m->nseg_max = (int)std::max(1L, std::min(4096L, (long)sms / ((long)cfg->B * cfg->H)));
        m->ws_per_unit =
            std::max(m->ws_per_unit, (size_t)m->nseg_max * titans::linear_scan_slot_floats(cfg->d, cfg->chunk));
    }
    m->ws_per_unit = (m->ws_per_unit + 255) & ~size_t(255);  // 1 KiB-aligned unit slices
    e = cudaMalloc(&m->ws, m->ws_per_unit * sizeof(float) * (size_t)cfg->B * cfg->H);
    if (e != cudaSuccess) {
        cudaFree(m->status);
        delete m;
        return cuda_fail(e, "allocating the workspace");
    }
    *out = m;
    return TITANS_OK;
}
}  // namespace

extern "C" {

titans_status_t titans_mem_init(const titans_mem_config* cfg, titans_mem_t* out) { return init_impl(cfg, 2, out); }

titans_status_t titans_mem_init_deep(const titans_mem_config* cfg, int layers, titans_mem_t* out) {
    return init_impl(cfg, layers, out);
}

titans_status_t titans_mem_destroy(titans_mem_t m) {
    if (!m) return fail(TITANS_EINVAL, "handle is NULL");
    for (cudaEvent_t e : m->ev) cudaEventDestroy(e);
    if (m->s_in) cudaStreamDestroy(m->s_in);
    if (m->s_out) cudaStreamDestroy(m->s_out);
    cudaFree(m->ws);
    cudaFree(m->status);
    delete m;
    return TITANS_OK;
}

int titans_mem_path(titans_mem_t m, int chunk, int step) {
    if (!m) return -1;
    if (step == 2) {  // titans_mem_backward
        if (m->layers > 2 || (m->cfg.flags & TITANS_FLAG_CHUNK_GATES) || chunk < 1 || chunk > m->cfg.chunk) return -1;
        return backward_tc_eligible(m->cfg, chunk) ? TITANS_PATH_TC_BACKWARD : TITANS_PATH_CUDA_CORES;
    }
    if (m->layers > 2) {
        if (step || chunk < 1 || chunk > m->cfg.chunk) return -1;
        return deep_tc_eligible(m->cfg, m->layers, chunk) ? TITANS_PATH_TC_DEEP : TITANS_PATH_DEEP_CUDA_CORES;
    }
    if (step) return m->cfg.d_hidden ? TITANS_PATH_STEP_CLUSTER : TITANS_PATH_CUDA_CORES;
    if (chunk < 1 || chunk > m->cfg.chunk) return -1;
    if (m->cfg.d_hidden == 0 && (m->cfg.flags & TITANS_FLAG_CHUNK_SCAN)) return TITANS_PATH_LINEAR_SCAN;
    if (tc_eligible(m->cfg, chunk)) return TITANS_PATH_TC_MLP64;
    return phased_eligible(m->cfg, chunk) ? TITANS_PATH_TC_PHASED : TITANS_PATH_CUDA_CORES;
}

}  // extern "C"

namespace {
// titans_mem_forward with the gates' row stride given separately (gate_ld >= T): the host-staged
// path reads the segments' gates in place from the full [units][T_total] arrays.
titans_status_t forward_impl(titans_mem_t m, const void* k, const void* q, const void* v, const float* alpha,
                             const float* eta, const float* theta, long gate_ld, long T, int chunk, float* W1,
                             float* W2, float* S1, float* S2, void* y, void* stream, const void* attn = nullptr) {
    if (!m) return fail(TITANS_EINVAL, "handle is NULL");
    if (m->layers > 2) return fail(TITANS_EINVAL, "a deep memory handle runs titans_mem_forward_deep");
    titans_status_t s = check_ptrs(m, k, q, v, alpha, eta, theta, W1, W2, S1, S2, y);
    if (s != TITANS_OK) return s;
    if (attn && !aligned16(attn)) return fail(TITANS_EINVAL, "attn is not 16-byte aligned");
    if (T < 1) return fail(TITANS_EINVAL, "T must be >= 1");
    if (T * (long)m->cfg.d >= (1L << 31)) return fail(TITANS_EUNSUPPORTED, "T * d must be below 2^31");
    if (chunk < 1 || chunk > m->cfg.chunk)
        return fail(TITANS_EUNSUPPORTED, "chunk must be in 1..config.chunk");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    titans::ForwardArgs a = make_args(m, k, q, v, alpha, eta, theta, T, chunk, W1, W2, S1, S2, y);
    a.gate_ld = gate_ld;
    a.attn = attn;
    cudaError_t e;
    if (tc_eligible(m->cfg, chunk)) {
        if (T >= (1L << 31) || a.units >= (1L << 31)) return fail(TITANS_EUNSUPPORTED, "T or units too large");
        CUtensorMap tk, tq, tv;
        if (!encode_tokens(&tk, k, T, a.units, chunk) || !encode_tokens(&tq, q, T, a.units, chunk) ||
            !encode_tokens(&tv, v, T, a.units, chunk))
            return fail(TITANS_ECUDA, "cuTensorMapEncodeTiled failed");
        e = titans::launch_chunk_tc_mlp64(a, tk, tq, tv, st);
    } else if (m->cfg.d_hidden == 0 && (m->cfg.flags & TITANS_FLAG_CHUNK_SCAN)) {
        e = titans::launch_linear_scan(a, m->nseg_max, st);
    } else if (phased_eligible(m->cfg, chunk)) {
        e = titans::launch_chunk_tc_phased(a, m->status + 2, st);
    } else {
        e = titans::launch_chunk_cuda_cores(a, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return TITANS_OK;
}

}  // namespace

extern "C" {

titans_status_t titans_mem_forward(titans_mem_t m, const void* k, const void* q, const void* v, const float* alpha,
                                   const float* eta, const float* theta, long T, int chunk, float* W1, float* W2,
                                   float* S1, float* S2, void* y, void* stream) {
    return forward_impl(m, k, q, v, alpha, eta, theta, gate_row(m, T, chunk), T, chunk, W1, W2, S1, S2, y, stream);
}

titans_status_t titans_mem_forward_gated(titans_mem_t m, const void* k, const void* q, const void* v,
                                         const float* alpha, const float* eta, const float* theta, long T, int chunk,
                                         float* W1, float* W2, float* S1, float* S2, const void* attn, void* o,
                                         void* stream) {
    if (!attn) return fail(TITANS_EINVAL, "attn is NULL");
    return forward_impl(m, k, q, v, alpha, eta, theta, gate_row(m, T, chunk), T, chunk, W1, W2, S1, S2, o, stream,
                        attn);
}

titans_status_t titans_mem_forward_deep(titans_mem_t m, const void* k, const void* q, const void* v,
                                        const float* alpha, const float* eta, const float* theta, long T, int chunk,
                                        float* W, float* S, const void* attn, void* y, void* stream) {
    if (!m) return fail(TITANS_EINVAL, "handle is NULL");
    if (!m->cfg.d_hidden) return fail(TITANS_EINVAL, "the deep forward needs an MLP memory (d_hidden > 0)");
    titans_status_t s = check_ptrs(m, k, q, v, alpha, eta, theta, W, W, S, S, y);
    if (s != TITANS_OK) return s;
    if (attn && !aligned16(attn)) return fail(TITANS_EINVAL, "attn is not 16-byte aligned");
    if (T < 1) return fail(TITANS_EINVAL, "T must be >= 1");
    if (T * (long)m->cfg.d >= (1L << 31)) return fail(TITANS_EUNSUPPORTED, "T * d must be below 2^31");
    if (chunk < 1 || chunk > m->cfg.chunk) return fail(TITANS_EUNSUPPORTED, "chunk must be in 1..config.chunk");
    titans::ForwardArgs a = make_args(m, k, q, v, alpha, eta, theta, T, chunk, W, nullptr, S, nullptr, y);
    a.attn = attn;
    cudaError_t e = m->layers > 2 && deep_tc_eligible(m->cfg, m->layers, chunk)
                        ? titans::launch_chunk_tc_deep(a, m->layers, m->status + 2, static_cast<cudaStream_t>(stream))
                        : titans::launch_chunk_deep_cuda_cores(a, m->layers, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return TITANS_OK;
}

titans_status_t titans_mem_forward_host(titans_mem_t m, const void* k, const void* q, const void* v,
                                        const float* alpha, const float* eta, const float* theta, long T, int chunk,
                                        float* W1, float* W2, float* S1, float* S2, void* y,
                                        const titans_device_buffers* dev, long t_seg, void* stream) {
    if (!m) return fail(TITANS_EINVAL, "handle is NULL");
    if (!dev) return fail(TITANS_EINVAL, "dev is NULL");
    const void* host[] = {k, q, v, alpha, eta, theta, y};
    const char* names[] = {"k", "q", "v", "alpha", "eta", "theta", "y"};
    for (int i = 0; i < 7; ++i)
        if (!host[i]) return fail(TITANS_EINVAL, std::string(names[i]) + " is NULL");
    titans_status_t s = check_ptrs(m, dev->k, dev->q, dev->v, dev->alpha, dev->eta, dev->theta, W1, W2, S1, S2,
                                   dev->y);
    if (s != TITANS_OK) return s;
    if (T < 1) return fail(TITANS_EINVAL, "T must be >= 1");
    if (chunk < 1 || chunk > m->cfg.chunk)
        return fail(TITANS_EUNSUPPORTED, "chunk must be in 1..config.chunk");
    if (t_seg < 0 || t_seg % chunk != 0) return fail(TITANS_EINVAL, "t_seg must be a non-negative multiple of chunk");
    // Automatic length: three times a sixteenth of T, in whole chunks (about five segments). On the
    // 128-unit, 4096-token stream it measured 4.36-4.40 ms per call against 4.50-4.52 ms with
    // sixteen segments: fewer, larger copies outweigh the longer last segment.
    if (t_seg == 0) t_seg = 3 * (((T + 15) / 16 + chunk - 1) / chunk * chunk);
    const long nseg = (T + t_seg - 1) / t_seg;
    if (nseg > 4096) return fail(TITANS_EINVAL, "more than 4096 segments: raise t_seg");
    int cur = -1;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (cur != m->device) return fail(TITANS_EINVAL, "the current device is not the handle's device");
    if (!m->s_in) {
        e = cudaStreamCreateWithFlags(&m->s_in, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&m->s_out, cudaStreamNonBlocking);
        if (e != cudaSuccess) return cuda_fail(e, "creating the copy streams");
    }
    while ((long)m->ev.size() < 2 + 2 * nseg) {
        cudaEvent_t ev;
        e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
        if (e != cudaSuccess) return cuda_fail(e, "creating events");
        m->ev.push_back(ev);
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t es = m->cfg.mode == TITANS_BF16 ? 2 : 4;  // token element size
    const size_t units = (size_t)m->cfg.B * m->cfg.H, d = (size_t)m->cfg.d;
    const size_t row_h = (size_t)T * d * es;  // one unit's host stream of k, q, v or y
    const long G = gate_row(m, T, chunk);     // one unit's gate row
    // The gates go over whole ([units][T], contiguous: one copy each, 12 B per head-token) and
    // the forward of each segment reads its columns in place. The tokens of segment i, [t0, t0 +
    // tn) of every unit, are packed on the device as [units][tn][d] at the offset of the segments
    // before it, so that each segment's k, q, v copy overlaps the previous segment's compute.
    e = cudaEventRecord(m->ev[0], st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(m->s_in, m->ev[0], 0);
    if (e != cudaSuccess) return cuda_fail(e, "ordering after the caller's stream");
    // From the first queued copy on, an error return first makes the caller's stream wait for
    // everything already queued on the copy streams (best effort), so that a caller who frees or
    // reuses the buffers once that stream is done cannot race with a copy still in flight.
    auto settle = [&](titans_status_t status) -> titans_status_t {
        if (cudaEventRecord(m->ev[0], m->s_in) == cudaSuccess) cudaStreamWaitEvent(st, m->ev[0], 0);
        if (cudaEventRecord(m->ev[1], m->s_out) == cudaSuccess) cudaStreamWaitEvent(st, m->ev[1], 0);
        return status;
    };
    {
        float* dg[3] = {dev->alpha, dev->eta, dev->theta};
        const float* hg[3] = {alpha, eta, theta};
        for (int j = 0; j < 3 && e == cudaSuccess; ++j)
            e = cudaMemcpyAsync(dg[j], hg[j], units * (size_t)G * 4, cudaMemcpyHostToDevice, m->s_in);
        if (e != cudaSuccess) return settle(cuda_fail(e, "copying the gates in"));
    }
    for (long i = 0; i < nseg; ++i) {
        const long t0 = i * t_seg, tn = std::min(t_seg, T - t0);
        const size_t tok_off = units * (size_t)t0 * d * es;
        char* dk[3] = {static_cast<char*>(dev->k) + tok_off, static_cast<char*>(dev->q) + tok_off,
                       static_cast<char*>(dev->v) + tok_off};
        const char* hk[3] = {static_cast<const char*>(k), static_cast<const char*>(q), static_cast<const char*>(v)};
        for (int j = 0; j < 3 && e == cudaSuccess; ++j)
            e = cudaMemcpy2DAsync(dk[j], (size_t)tn * d * es, hk[j] + (size_t)t0 * d * es, row_h, (size_t)tn * d * es,
                                  units, cudaMemcpyHostToDevice, m->s_in);
        if (e == cudaSuccess) e = cudaEventRecord(m->ev[2 + 2 * i], m->s_in);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, m->ev[2 + 2 * i], 0);
        if (e != cudaSuccess) return settle(cuda_fail(e, "copying a segment in"));
        char* dy = static_cast<char*>(dev->y) + tok_off;
        const long g0 = G == T ? t0 : t0 / chunk;  // the segment's first gate column
        s = forward_impl(m, dk[0], dk[1], dk[2], dev->alpha + g0, dev->eta + g0, dev->theta + g0, G, tn, chunk, W1,
                         W2, S1, S2, dy, stream);
        if (s != TITANS_OK) return settle(s);
        e = cudaEventRecord(m->ev[3 + 2 * i], st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(m->s_out, m->ev[3 + 2 * i], 0);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(static_cast<char*>(y) + (size_t)t0 * d * es, row_h, dy, (size_t)tn * d * es,
                                  (size_t)tn * d * es, units, cudaMemcpyDeviceToHost, m->s_out);
        if (e != cudaSuccess) return settle(cuda_fail(e, "copying a segment out"));
    }
    e = cudaEventRecord(m->ev[1], m->s_out);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, m->ev[1], 0);
    if (e != cudaSuccess) return settle(cuda_fail(e, "ordering the caller's stream after the copies"));
    return TITANS_OK;
}

}  // extern "C"

namespace {
titans_status_t step_impl(titans_mem_t m, const void* k, const void* q, const void* v, const float* alpha,
                          const float* eta, const float* theta, float* W1, float* W2, float* S1, float* S2, void* y,
                          void* stream, const void* attn) {
    if (!m) return fail(TITANS_EINVAL, "handle is NULL");
    if (m->layers > 2) return fail(TITANS_EUNSUPPORTED, "no decode step for a deep memory handle");
    titans_status_t s = check_ptrs(m, k, q, v, alpha, eta, theta, W1, W2, S1, S2, y);
    if (s != TITANS_OK) return s;
    if (attn && !aligned16(attn)) return fail(TITANS_EINVAL, "attn is not 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    titans::ForwardArgs a = make_args(m, k, q, v, alpha, eta, theta, 1, 1, W1, W2, S1, S2, y);
    a.attn = attn;
    cudaError_t e = m->cfg.d_hidden ? titans::launch_step_cluster(a, st) : titans::launch_chunk_cuda_cores(a, st);
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return TITANS_OK;
}
}  // namespace

extern "C" {

titans_status_t titans_mem_step(titans_mem_t m, const void* k, const void* q, const void* v, const float* alpha,
                                const float* eta, const float* theta, float* W1, float* W2, float* S1, float* S2,
                                void* y, void* stream) {
    return step_impl(m, k, q, v, alpha, eta, theta, W1, W2, S1, S2, y, stream, nullptr);
}

titans_status_t titans_mem_step_gated(titans_mem_t m, const void* k, const void* q, const void* v,
                                      const float* alpha, const float* eta, const float* theta, float* W1, float* W2,
                                      float* S1, float* S2, const void* attn, void* o, void* stream) {
    if (!attn) return fail(TITANS_EINVAL, "attn is NULL");
    return step_impl(m, k, q, v, alpha, eta, theta, W1, W2, S1, S2, o, stream, attn);
}

size_t titans_mem_backward_workspace_bytes(titans_mem_t m, long T, int chunk) {
    if (!m || T < 1 || chunk < 1) return 0;
    size_t f = m->cfg.d_hidden ? titans::mlp_backward_ws_floats(m->cfg.d, m->cfg.d_hidden, T, chunk)
                               : titans::linear_backward_ws_floats(m->cfg.d, T, chunk);
    if (backward_tc_eligible(m->cfg, chunk))
        f = std::max(f, (titans::mlp_backward_tc_ws_bytes(T, chunk) + sizeof(float) - 1) / sizeof(float));
    const size_t per_unit = (f + 63) & ~size_t(63);
    const size_t units = (size_t)m->cfg.B * m->cfg.H;
    // the tensor-core backward runs the forward once on a copy of the initial state, kept after
    // the units' slices: W1, W2, S1, S2 [units][h * d] each
    const size_t fwd_state = backward_tc_eligible(m->cfg, chunk)
                                 ? 4 * units * (size_t)m->cfg.d * m->cfg.d_hidden * sizeof(float)
                                 : 0;
    return per_unit * sizeof(float) * units + fwd_state;
}

titans_status_t titans_mem_backward(titans_mem_t m, const void* k, const void* q, const void* v, const float* alpha,
                                    const float* eta, const float* theta, long T, int chunk, const float* W1,
                                    const float* W2, const float* S1, const float* S2, const void* dy,
                                    const float* dW1, const float* dW2, const float* dS1, const float* dS2, void* dk,
                                    void* dq, void* dv, float* dalpha, float* deta, float* dtheta, float* dW1_0,
                                    float* dW2_0, float* dS1_0, float* dS2_0, void* workspace, size_t workspace_bytes,
                                    void* stream) {
    if (!m) return fail(TITANS_EINVAL, "handle is NULL");
    if (m->layers > 2) return fail(TITANS_EUNSUPPORTED, "the backward is built for the linear and the 2-layer memory");
    if (m->cfg.flags & TITANS_FLAG_CHUNK_GATES) return fail(TITANS_EUNSUPPORTED, "the backward takes per-token gates");
    const bool mlp = m->cfg.d_hidden != 0;
    const void* req[] = {k, q, v, W1, S1, dy, dk, dq, dv, dW1_0, dS1_0, workspace};
    const char* names[] = {"k", "q", "v", "W1", "S1", "dy", "dk", "dq", "dv", "dW1_0", "dS1_0", "workspace"};
    for (int i = 0; i < 12; ++i) {
        if (!req[i]) return fail(TITANS_EINVAL, std::string(names[i]) + " is NULL");
        if (!aligned16(req[i])) return fail(TITANS_EINVAL, std::string(names[i]) + " is not 16-byte aligned");
    }
    if (mlp) {
        const void* req2[] = {W2, S2, dW2_0, dS2_0};
        for (const void* p : req2)
            if (!p || !aligned16(p)) return fail(TITANS_EINVAL, "W2, S2, dW2_0, dS2_0 must be non-NULL and 16-byte aligned");
    }
    const float* g4[] = {alpha, eta, theta, dalpha, deta, dtheta};
    for (const float* p : g4)
        if (!p || (reinterpret_cast<uintptr_t>(p) & 3u))
            return fail(TITANS_EINVAL, "the gates and their gradients must be non-NULL and 4-byte aligned");
    if (T < 1) return fail(TITANS_EINVAL, "T must be >= 1");
    if (T * (long)m->cfg.d >= (1L << 31)) return fail(TITANS_EUNSUPPORTED, "T * d must be below 2^31");
    if (chunk < 1 || chunk > m->cfg.chunk) return fail(TITANS_EUNSUPPORTED, "chunk must be in 1..config.chunk");
    const size_t need = titans_mem_backward_workspace_bytes(m, T, chunk);
    if (workspace_bytes < need)
        return fail(TITANS_EINVAL, "workspace smaller than titans_mem_backward_workspace_bytes(): " +
                                       std::to_string(workspace_bytes) + " < " + std::to_string(need));
    const long units = (long)m->cfg.B * m->cfg.H;
    cudaError_t e = cudaSuccess;
    if (mlp) {
        titans::MlpBackwardArgs b{};
        b.d = m->cfg.d;
        b.h = m->cfg.d_hidden;
        b.chunk = chunk;
        b.units = units;
        b.T = T;
        b.bf16 = m->cfg.mode == TITANS_BF16;
        b.k = k;
        b.q = q;
        b.v = v;
        b.dy = dy;
        b.alpha = alpha;
        b.eta = eta;
        b.theta = theta;
        b.W1 = W1;
        b.W2 = W2;
        b.S1 = S1;
        b.S2 = S2;
        b.dW1 = dW1;
        b.dW2 = dW2;
        b.dS1 = dS1;
        b.dS2 = dS2;
        b.dk = dk;
        b.dq = dq;
        b.dv = dv;
        b.dalpha = dalpha;
        b.deta = deta;
        b.dtheta = dtheta;
        b.dW1_0 = dW1_0;
        b.dW2_0 = dW2_0;
        b.dS1_0 = dS1_0;
        b.dS2_0 = dS2_0;
        b.ws = static_cast<float*>(workspace);
        b.status = m->status;
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        if (backward_tc_eligible(m->cfg, chunk)) {
            // The forward with checkpoints: the tensor-core chunk kernel runs on a copy of the initial
            // state and writes every chunk-start state into the units' workspace slices (y goes to
            // dk, which the backward overwrites).
            const size_t hd = (size_t)m->cfg.d * m->cfg.d_hidden;
            const size_t fwd_state = 4 * (size_t)units * hd * sizeof(float);
            b.ws_per_unit = (need - fwd_state) / sizeof(float) / (size_t)units;
            float* sw = reinterpret_cast<float*>(static_cast<char*>(workspace) + (need - fwd_state));
            float* sW[4] = {sw, sw + units * hd, sw + 2 * units * hd, sw + 3 * units * hd};
            const float* src[4] = {W1, W2, S1, S2};
            for (int i = 0; i < 4 && e == cudaSuccess; ++i)
                e = cudaMemcpyAsync(sW[i], src[i], (size_t)units * hd * sizeof(float), cudaMemcpyDeviceToDevice, st);
            if (e != cudaSuccess) return cuda_fail(e, "copying the initial state");
            CUtensorMap tk, tq, tv;
            if (!encode_tokens(&tk, k, T, units, chunk) || !encode_tokens(&tq, q, T, units, chunk) ||
                !encode_tokens(&tv, v, T, units, chunk))
                return fail(TITANS_ECUDA, "cuTensorMapEncodeTiled failed");
            titans::ForwardArgs a = make_args(m, k, q, v, alpha, eta, theta, T, chunk, sW[0], sW[1], sW[2], sW[3], dk);
            a.ckpt = reinterpret_cast<float*>(static_cast<char*>(workspace) + titans::mlp_backward_tc_ckpt_offset());
            a.ckpt_unit_stride = b.ws_per_unit;
            e = titans::launch_chunk_tc_mlp64(a, tk, tq, tv, st);
            if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
            b.ckpt_ready = true;
            e = titans::launch_mlp_backward_tc(b, st);
        } else {
            b.ws_per_unit = need / sizeof(float) / (size_t)units;
            e = titans::launch_mlp_backward(b, st);
        }
    } else {
        titans::LinearBackwardArgs b{};
        b.d = m->cfg.d;
        b.chunk = chunk;
        b.units = units;
        b.T = T;
        b.bf16 = m->cfg.mode == TITANS_BF16;
        b.k = k;
        b.q = q;
        b.v = v;
        b.dy = dy;
        b.alpha = alpha;
        b.eta = eta;
        b.theta = theta;
        b.W0 = W1;
        b.S0 = S1;
        b.dWT = dW1;
        b.dST = dS1;
        b.dk = dk;
        b.dq = dq;
        b.dv = dv;
        b.dalpha = dalpha;
        b.deta = deta;
        b.dtheta = dtheta;
        b.dW0 = dW1_0;
        b.dS0 = dS1_0;
        b.ws = static_cast<float*>(workspace);
        b.ws_per_unit = need / sizeof(float) / (size_t)units;
        e = titans::launch_linear_backward(b, static_cast<cudaStream_t>(stream));
    }
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
        char buf[192];
        snprintf(buf, sizeof buf,
                 "device status 0x%x (1: TMA wait timed out, 2: MMA wait timed out, 4: grid barrier timed out, "
                 "8: a bounds check of the debug build failed)", h);
        return fail(TITANS_EDEVICE, buf);
    }
    return TITANS_OK;
}

}  // extern "C"
