// Cross-chunk scan of the linear memory M(x) = W x ("Titans: Learning to Memorize at Test Time":
// walk-through sec. 3.2; the German summary's "Parallelisiertes Training" and the tencent review
// name parallel associative scans for the recurrent part).
//
// One chunk of the linear memory is an affine map of the row state X = [W | S] (d x 2d):
//   X' = X M + N,  M = [[A I - 2 K^T C K, -2 K^T D K], [sigma I, E I]],  N = [2 V^T C K, 2 V^T D K],
// (K, V the chunk's keys and values as rows, C = diag(c), D = diag(d) from the gate scan), so the
// chunks of a stream combine associatively and a single long stream can use many SMs:
//   1. compose: each segment of G chunks composes its chunks' maps. Appending a chunk to a composed
//      map (M, N) multiplies every row of [M; N] by the chunk's map, which is the ordinary chunk
//      update applied to a 3d-row state whose first 2d rows (M) see v = 0 and last d rows (N) see
//      v: started from [I; 0], one CTA per (unit, segment);
//   2. scan: per unit, X_{s+1} = X_s M_s + N_s over the segments, in order (one CTA per unit);
//   3. run: each segment runs its chunks from X_s, writing y_t = W q_t with the chunk-start W (one
//      CTA per (unit, segment)); the last segment hands the final W, S back.
// fp32 arithmetic on CUDA cores; k, q, v, y in fp32 or bf16.
#include <cuda_bf16.h>

#include <atomic>
#include <cstdint>

#include "kernels.h"

namespace titans {

namespace {

__device__ __forceinline__ float ldx(const float* p) { return *p; }
__device__ __forceinline__ float ldx(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void stx(float* p, float v) { *p = v; }
__device__ __forceinline__ void stx(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

constexpr int kScanThreads = 1024;
constexpr int kScanMaxChunk = 128;

// Per (unit, segment) workspace slot, in floats: R [3d][2d], P [3d][n], X [d][2d], G [n][d], and a
// second map buffer R2 [3d][2d] for the tree scan over segments.
__host__ __device__ inline size_t slot_floats(int d, int n) {
    return (size_t)6 * d * d + (size_t)3 * d * n + (size_t)2 * d * d + (size_t)n * d + (size_t)6 * d * d;
}
__host__ __device__ inline size_t slot_r2(int d, int n) {
    return (size_t)6 * d * d + (size_t)3 * d * n + (size_t)2 * d * d + (size_t)n * d;
}

// The chunk's gate scan (division-free suffix scan) into shared memory: c, d, and A, E, sigma.
__device__ void chunk_scan(const float* alpha, const float* eta, const float* theta, long t0, int n, int chunk,
                           int chunk_gates, float* s_a, float* s_e, float* s_t, float* s_c, float* s_d, float* s_scal) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const long gi = chunk_gates ? t0 / chunk : t0 + i;
        s_a[i] = alpha[gi];
        s_e[i] = eta[gi];
        s_t[i] = theta[gi];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float Pr = 1.f, Qr = 1.f, r_next = 0.f;
        for (int j = n - 1; j >= 0; --j) {
            const float r = Pr + (j + 1 < n ? s_e[j + 1] * r_next : 0.f);
            s_c[j] = s_t[j] * r;
            s_d[j] = s_t[j] * Qr;
            r_next = r;
            Pr *= 1.f - s_a[j];
            Qr *= s_e[j];
        }
        s_scal[0] = Pr;
        s_scal[1] = Qr;
        s_scal[2] = s_e[0] * r_next;
    }
    __syncthreads();
}

}  // namespace

size_t linear_scan_slot_floats(int d, int n) { return slot_floats(d, n); }

// 1. compose the maps of segment s of unit u (blockIdx = u * nseg + s).
template <typename Tin>
__global__ void __launch_bounds__(kScanThreads) linear_scan_compose(
    int d, long T, long gate_ld, int chunk, int chunk_gates, int nseg, int G, const Tin* __restrict__ k,
    const Tin* __restrict__ v, const float* __restrict__ alpha, const float* __restrict__ eta,
    const float* __restrict__ theta, float* __restrict__ ws, size_t ws_per_unit) {
    __shared__ float s_a[kScanMaxChunk], s_e[kScanMaxChunk], s_t[kScanMaxChunk], s_c[kScanMaxChunk],
        s_d[kScanMaxChunk], s_scal[3];
    const long u = blockIdx.x / nseg;
    const int s = blockIdx.x % nseg, tid = threadIdx.x;
    float* R = ws + u * ws_per_unit + (size_t)s * slot_floats(d, chunk);
    float* P = R + (size_t)6 * d * d;
    const int d2 = 2 * d, rows = 3 * d;
    for (int idx = tid; idx < rows * d2; idx += blockDim.x) {
        const int r = idx / d2, col = idx % d2;
        R[idx] = (r < d2 && col == r) ? 1.f : 0.f;
    }
    __syncthreads();
    k += u * T * d;
    v += u * T * d;
    alpha += u * gate_ld;
    eta += u * gate_ld;
    theta += u * gate_ld;
    const int nch = (int)((T + chunk - 1) / chunk);
    const int c1 = min(nch, (s + 1) * G);
    for (int c = s * G; c < c1; ++c) {
        const long t0 = (long)c * chunk;
        const int n = (int)min((long)chunk, T - t0);
        chunk_scan(alpha, eta, theta, t0, n, chunk, chunk_gates, s_a, s_e, s_t, s_c, s_d, s_scal);
        const float An = s_scal[0], En = s_scal[1], sig = s_scal[2];
        const Tin* K = k + t0 * d;
        const Tin* V = v + t0 * d;
        // P[r][t] = (row r of the W part) . k_t  - (v_t's component for the N rows)
        for (int idx = tid; idx < rows * n; idx += blockDim.x) {
            const int r = idx / n, t = idx % n;
            float p = 0.f;
            const float* Rr = R + (size_t)r * d2;
            for (int m = 0; m < d; ++m) p += Rr[m] * ldx(K + (size_t)t * d + m);
            if (r >= d2) p -= ldx(V + (size_t)t * d + (r - d2));
            P[idx] = p;
        }
        __syncthreads();
        for (int idx = tid; idx < rows * d; idx += blockDim.x) {
            const int r = idx / d, m = idx % d;
            float uc = 0.f, ud = 0.f;
            for (int t = 0; t < n; ++t) {
                const float g = P[(size_t)r * n + t] * ldx(K + (size_t)t * d + m);
                uc += s_c[t] * g;
                ud += s_d[t] * g;
            }
            float* Rr = R + (size_t)r * d2;
            const float w = Rr[m], sv = Rr[d + m];
            Rr[m] = An * w + sig * sv - 2.f * uc;
            Rr[d + m] = En * sv - 2.f * ud;
        }
        __syncthreads();
    }
}

// 1'. The same composition with the map, the chunk's keys and the products in shared memory (d = 64):
// R [3d][2d], P [3d][n], the keys [n][d + 1] (one padding column so that a warp reading one column
// of 16 or more key rows does not hit one bank), 96 KB + about 1 KB per token of the chunk.
constexpr int kComposeSmemMaxChunk = 64;  // chunks up to 64 tokens: 160 KB of shared memory at most
__host__ __device__ inline size_t compose_smem_bytes(int chunk) {
    constexpr int d = 64;
    return ((size_t)6 * d * d + (size_t)3 * d * chunk + (size_t)chunk * (d + 1)) * sizeof(float);
}

template <typename Tin>
__global__ void __launch_bounds__(kScanThreads) linear_scan_compose_smem(
    long T, long gate_ld, int chunk, int chunk_gates, int nseg, int G, const Tin* __restrict__ k,
    const Tin* __restrict__ v, const float* __restrict__ alpha, const float* __restrict__ eta,
    const float* __restrict__ theta, float* __restrict__ ws, size_t ws_per_unit) {
    constexpr int d = 64, d2 = 128, rows = 192;
    __shared__ float s_a[kScanMaxChunk], s_e[kScanMaxChunk], s_t[kScanMaxChunk], s_c[kScanMaxChunk],
        s_d[kScanMaxChunk], s_scal[3];
    extern __shared__ float smf[];
    float* sR = smf;                         // [3d][2d]
    float* sP = sR + rows * d2;              // [3d][n]
    float* sK = sP + (size_t)rows * chunk;   // [n][d + 1]
    const long u = blockIdx.x / nseg;
    const int s = blockIdx.x % nseg, tid = threadIdx.x;
    float* R = ws + u * ws_per_unit + (size_t)s * slot_floats(d, chunk);
    for (int idx = tid; idx < rows * d2; idx += blockDim.x) {
        const int r = idx / d2, col = idx % d2;
        sR[idx] = (r < d2 && col == r) ? 1.f : 0.f;
    }
    k += u * T * d;
    v += u * T * d;
    alpha += u * gate_ld;
    eta += u * gate_ld;
    theta += u * gate_ld;
    const int nch = (int)((T + chunk - 1) / chunk);
    const int c1 = min(nch, (s + 1) * G);
    for (int c = s * G; c < c1; ++c) {
        const long t0 = (long)c * chunk;
        const int n = (int)min((long)chunk, T - t0);
        chunk_scan(alpha, eta, theta, t0, n, chunk, chunk_gates, s_a, s_e, s_t, s_c, s_d, s_scal);
        const float An = s_scal[0], En = s_scal[1], sig = s_scal[2];
        const Tin* K = k + t0 * d;
        const Tin* V = v + t0 * d;
        for (int idx = tid; idx < n * d; idx += blockDim.x) sK[(idx / d) * (d + 1) + idx % d] = ldx(K + idx);
        __syncthreads();
        // P[r][t] = (row r of the W part) . k_t  - (v_t's component for the N rows)
        for (int idx = tid; idx < rows * n; idx += blockDim.x) {
            const int r = idx / n, t = idx % n;
            float p = 0.f;
            const float* Rr = sR + r * d2;
            const float* Kt = sK + t * (d + 1);
#pragma unroll 8
            for (int m = 0; m < d; ++m) p = fmaf(Rr[m], Kt[m], p);
            if (r >= d2) p -= ldx(V + (size_t)t * d + (r - d2));
            sP[r * n + t] = p;
        }
        __syncthreads();
        for (int idx = tid; idx < rows * d; idx += blockDim.x) {
            const int r = idx / d, m = idx % d;
            float uc = 0.f, ud = 0.f;
            for (int t = 0; t < n; ++t) {
                const float g = sP[r * n + t] * sK[t * (d + 1) + m];
                uc = fmaf(s_c[t], g, uc);
                ud = fmaf(s_d[t], g, ud);
            }
            float* Rr = sR + r * d2;
            const float w = Rr[m], sv = Rr[d + m];
            Rr[m] = An * w + sig * sv - 2.f * uc;
            Rr[d + m] = En * sv - 2.f * ud;
        }
        __syncthreads();
    }
    for (int i = tid; i < rows * d2 / 4; i += blockDim.x)
        reinterpret_cast<float4*>(R)[i] = reinterpret_cast<const float4*>(sR)[i];
}

// 2. per unit: X_0 = [W | S], X_{s+1} = X_s M_s + N_s (M_s = R_s rows 0..2d-1, N_s = rows 2d..3d-1).
__global__ void __launch_bounds__(kScanThreads) linear_scan_segments(int d, int chunk, int nseg_used, int nseg,
                                                                   const float* __restrict__ W,
                                                                   const float* __restrict__ S,
                                                                   float* __restrict__ ws, size_t ws_per_unit) {
    const long u = blockIdx.x;
    const int d2 = 2 * d;
    const size_t slot = slot_floats(d, chunk);
    float* base = ws + u * ws_per_unit;
    auto Xof = [&](int s) { return base + (size_t)s * slot + (size_t)6 * d * d + (size_t)3 * d * chunk; };
    float* X0 = Xof(0);
    for (int idx = threadIdx.x; idx < d * d2; idx += blockDim.x) {
        const int i = idx / d2, j = idx % d2;
        X0[idx] = j < d ? W[u * d * d + (size_t)i * d + j] : S[u * d * d + (size_t)i * d + (j - d)];
    }
    __syncthreads();
    for (int s = 0; s + 1 < nseg_used; ++s) {
        const float* Xs = Xof(s);
        const float* R = base + (size_t)s * slot;
        float* Xn = Xof(s + 1);
        for (int idx = threadIdx.x; idx < d * d2; idx += blockDim.x) {
            const int i = idx / d2, j = idx % d2;
            float acc = R[(size_t)(d2 + i) * d2 + j];  // N_s[i][j]
            for (int r = 0; r < d2; ++r) acc += Xs[(size_t)i * d2 + r] * R[(size_t)r * d2 + j];
            Xn[idx] = acc;
        }
        __syncthreads();
    }
    (void)nseg;
}

// 2'. The same scan with the state and each segment's map in shared memory (d = 64: the map R_s
// [3d][2d] and two state buffers [d][2d], 160 KB): every step reads its operands from shared memory
// instead of L2, and the next segment's map is copied in while nothing else waits on it.
constexpr int kSegSmemD = 64;
constexpr int kTreeMinSegments = 16;  // below this the sequential scan (one CTA per unit) is as fast
constexpr size_t kSegSmemBytes = (size_t)(6 * kSegSmemD * kSegSmemD + 4 * kSegSmemD * kSegSmemD) * sizeof(float);

static_assert(kScanThreads == 1024, "the shared-memory segment scan maps 1024 threads onto d x 2d = 64 x 128");
__global__ void __launch_bounds__(kScanThreads) linear_scan_segments_smem(int chunk, int nseg_used,
                                                                        const float* __restrict__ W,
                                                                        const float* __restrict__ S,
                                                                        float* __restrict__ ws, size_t ws_per_unit) {
    constexpr int d = kSegSmemD, d2 = 2 * kSegSmemD;
    extern __shared__ float smf[];
    float* sR = smf;               // [3d][2d]: M_s rows 0..2d-1, N_s rows 2d..3d-1
    float* sX0 = sR + 3 * d * d2;  // [d][2d] state buffers
    float* sX1 = sX0 + d * d2;
    const long u = blockIdx.x;
    const size_t slot = slot_floats(d, chunk);
    float* base = ws + u * ws_per_unit;
    auto Xof = [&](int s) { return base + (size_t)s * slot + (size_t)6 * d * d + (size_t)3 * d * chunk; };
    float* X0 = Xof(0);
    for (int idx = threadIdx.x; idx < d * d2; idx += blockDim.x) {
        const int i = idx / d2, j = idx % d2;
        const float x = j < d ? W[u * d * d + (size_t)i * d + j] : S[u * d * d + (size_t)i * d + (j - d)];
        X0[idx] = x;
        sX0[idx] = x;
    }
    float* cur = sX0;
    float* nxt = sX1;
    for (int s = 0; s + 1 < nseg_used; ++s) {
        __syncthreads();  // the previous step's reads of sR are done
        const float4* R4 = reinterpret_cast<const float4*>(base + (size_t)s * slot);
        for (int i = threadIdx.x; i < 3 * d * d2 / 4; i += blockDim.x) reinterpret_cast<float4*>(sR)[i] = R4[i];
        __syncthreads();
        float* Xn = Xof(s + 1);
        // thread: rows i0 and i0 + 32, columns 4 j4 .. 4 j4 + 3 (1024 threads x 8 outputs = d x 2d)
        const int i0 = threadIdx.x >> 5, j4 = threadIdx.x & 31;
        float4 a0 = *reinterpret_cast<const float4*>(sR + (d2 + i0) * d2 + 4 * j4);  // N_s rows
        float4 a1 = *reinterpret_cast<const float4*>(sR + (d2 + i0 + 32) * d2 + 4 * j4);
#pragma unroll 8
        for (int r = 0; r < d2; ++r) {
            const float x0 = cur[i0 * d2 + r], x1 = cur[(i0 + 32) * d2 + r];
            const float4 m = *reinterpret_cast<const float4*>(sR + r * d2 + 4 * j4);
            a0.x = fmaf(x0, m.x, a0.x);
            a0.y = fmaf(x0, m.y, a0.y);
            a0.z = fmaf(x0, m.z, a0.z);
            a0.w = fmaf(x0, m.w, a0.w);
            a1.x = fmaf(x1, m.x, a1.x);
            a1.y = fmaf(x1, m.y, a1.y);
            a1.z = fmaf(x1, m.z, a1.z);
            a1.w = fmaf(x1, m.w, a1.w);
        }
        *reinterpret_cast<float4*>(nxt + i0 * d2 + 4 * j4) = a0;
        *reinterpret_cast<float4*>(nxt + (i0 + 32) * d2 + 4 * j4) = a1;
        *reinterpret_cast<float4*>(Xn + i0 * d2 + 4 * j4) = a0;
        *reinterpret_cast<float4*>(Xn + (i0 + 32) * d2 + 4 * j4) = a1;
        float* t = cur;
        cur = nxt;
        nxt = t;
    }
}

// 2''. The scan over segments as a tree (d = 64): Hillis-Steele levels, each composing every map
// with the one 2^level segments before it, so that after ceil(log2 S) levels map s is
// F_s o ... o F_0; then X_{s+1} = X_0 M + N for every segment at once. Composition, X -> (X M_a +
// N_a) M_b + N_b: R_out = R_a M_b + [0; N_b] with R = [M; N] ([3d][2d]); one CTA per (unit,
// segment), both maps in shared memory (160 KB), 6 x 4 outputs per thread.
constexpr size_t kTreeSmemBytes = (size_t)(6 * 64 * 64 + 4 * 64 * 64) * sizeof(float);

__global__ void __launch_bounds__(kScanThreads) linear_scan_tree_level(int chunk, int nseg_used, int step, int src2,
                                                                     float* __restrict__ ws, size_t ws_per_unit) {
    constexpr int d = 64, d2 = 128, rows = 192;
    extern __shared__ float smf[];
    float* sA = smf;              // R_a [3d][2d]
    float* sM = sA + rows * d2;   // M_b [2d][2d]
    const long u = blockIdx.x / nseg_used;
    const int s = blockIdx.x % nseg_used, tid = threadIdx.x;
    const size_t slot = slot_floats(d, chunk), r2 = slot_r2(d, chunk);
    float* base = ws + u * ws_per_unit;
    auto map_in = [&](int seg) { return base + (size_t)seg * slot + (src2 ? r2 : 0); };
    float* out = base + (size_t)s * slot + (src2 ? 0 : r2);
    const float* Rb = map_in(s);
    if (s < step) {  // nothing 2^level segments back: the map carries over
        for (int i = tid; i < rows * d2 / 4; i += blockDim.x)
            reinterpret_cast<float4*>(out)[i] = reinterpret_cast<const float4*>(Rb)[i];
        return;
    }
    const float* Ra = map_in(s - step);
    for (int i = tid; i < rows * d2 / 4; i += blockDim.x)
        reinterpret_cast<float4*>(sA)[i] = reinterpret_cast<const float4*>(Ra)[i];
    for (int i = tid; i < d2 * d2 / 4; i += blockDim.x)
        reinterpret_cast<float4*>(sM)[i] = reinterpret_cast<const float4*>(Rb)[i];
    __syncthreads();
    const int i0 = tid >> 5, j4 = tid & 31;  // rows i0 + 32 q (q < 6), columns 4 j4 .. 4 j4 + 3
    float4 acc[6];
#pragma unroll
    for (int qr = 0; qr < 6; ++qr) {
        const int r = i0 + 32 * qr;  // N_b joins the N rows (r >= 2d)
        acc[qr] = r >= d2 ? *reinterpret_cast<const float4*>(Rb + (size_t)r * d2 + 4 * j4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll 4
    for (int k = 0; k < d2; ++k) {
        const float4 m = *reinterpret_cast<const float4*>(sM + k * d2 + 4 * j4);
#pragma unroll
        for (int qr = 0; qr < 6; ++qr) {
            const float a = sA[(i0 + 32 * qr) * d2 + k];
            acc[qr].x = fmaf(a, m.x, acc[qr].x);
            acc[qr].y = fmaf(a, m.y, acc[qr].y);
            acc[qr].z = fmaf(a, m.z, acc[qr].z);
            acc[qr].w = fmaf(a, m.w, acc[qr].w);
        }
    }
#pragma unroll
    for (int qr = 0; qr < 6; ++qr) *reinterpret_cast<float4*>(out + (size_t)(i0 + 32 * qr) * d2 + 4 * j4) = acc[qr];
}

// X_0 = [W | S] into slot 0; X_{s+1} = X_0 M + N with the composed map s, for s < S - 1.
__global__ void __launch_bounds__(kScanThreads) linear_scan_tree_apply(int chunk, int nseg_used, int src2,
                                                                     const float* __restrict__ W,
                                                                     const float* __restrict__ S,
                                                                     float* __restrict__ ws, size_t ws_per_unit) {
    constexpr int d = 64, d2 = 128;
    extern __shared__ float smf[];
    float* sX = smf;             // X_0 [d][2d]
    float* sM = sX + d * d2;     // M [2d][2d]
    const long u = blockIdx.x / nseg_used;
    const int s = blockIdx.x % nseg_used, tid = threadIdx.x;
    const size_t slot = slot_floats(d, chunk);
    float* base = ws + u * ws_per_unit;
    auto Xof = [&](int seg) { return base + (size_t)seg * slot + (size_t)6 * d * d + (size_t)3 * d * chunk; };
    for (int idx = tid; idx < d * d2; idx += blockDim.x) {
        const int i = idx / d2, j = idx % d2;
        sX[idx] = j < d ? W[u * d * d + (size_t)i * d + j] : S[u * d * d + (size_t)i * d + (j - d)];
    }
    if (s == 0)
        for (int idx = tid; idx < d * d2; idx += blockDim.x) Xof(0)[idx] = sX[idx];
    if (s + 1 >= nseg_used) return;
    const float* R = base + (size_t)s * slot + (src2 ? slot_r2(d, chunk) : 0);
    for (int i = tid; i < d2 * d2 / 4; i += blockDim.x)
        reinterpret_cast<float4*>(sM)[i] = reinterpret_cast<const float4*>(R)[i];
    __syncthreads();
    const int i0 = tid >> 5, j4 = tid & 31;
    float4 a0 = *reinterpret_cast<const float4*>(R + (size_t)(d2 + i0) * d2 + 4 * j4);
    float4 a1 = *reinterpret_cast<const float4*>(R + (size_t)(d2 + i0 + 32) * d2 + 4 * j4);
#pragma unroll 8
    for (int r = 0; r < d2; ++r) {
        const float x0 = sX[i0 * d2 + r], x1 = sX[(i0 + 32) * d2 + r];
        const float4 m = *reinterpret_cast<const float4*>(sM + r * d2 + 4 * j4);
        a0.x = fmaf(x0, m.x, a0.x);
        a0.y = fmaf(x0, m.y, a0.y);
        a0.z = fmaf(x0, m.z, a0.z);
        a0.w = fmaf(x0, m.w, a0.w);
        a1.x = fmaf(x1, m.x, a1.x);
        a1.y = fmaf(x1, m.y, a1.y);
        a1.z = fmaf(x1, m.z, a1.z);
        a1.w = fmaf(x1, m.w, a1.w);
    }
    float* Xn = Xof(s + 1);
    *reinterpret_cast<float4*>(Xn + i0 * d2 + 4 * j4) = a0;
    *reinterpret_cast<float4*>(Xn + (i0 + 32) * d2 + 4 * j4) = a1;
}

// 3. run segment s of unit u from X_s: y for its tokens; the last segment writes the final W, S.
template <typename Tin>
__global__ void __launch_bounds__(kScanThreads) linear_scan_run(
    int d, long T, long gate_ld, int chunk, int chunk_gates, int nseg_used, int G, const Tin* __restrict__ k,
    const Tin* __restrict__ q, const Tin* __restrict__ v, const float* __restrict__ alpha,
    const float* __restrict__ eta, const float* __restrict__ theta, float* __restrict__ Wout,
    float* __restrict__ Sout, Tin* __restrict__ y, const Tin* __restrict__ attn, float* __restrict__ ws,
    size_t ws_per_unit) {
    __shared__ float s_a[kScanMaxChunk], s_e[kScanMaxChunk], s_t[kScanMaxChunk], s_c[kScanMaxChunk],
        s_d[kScanMaxChunk], s_scal[3];
    const long u = blockIdx.x / nseg_used;
    const int s = blockIdx.x % nseg_used, tid = threadIdx.x, d2 = 2 * d;
    float* slotp = ws + u * ws_per_unit + (size_t)s * slot_floats(d, chunk);
    float* X = slotp + (size_t)6 * d * d + (size_t)3 * d * chunk;  // [d][2d]: W | S, updated in place
    float* Ge = X + (size_t)2 * d * d;                                // [n][d]
    k += u * T * d;
    q += u * T * d;
    v += u * T * d;
    y += u * T * d;
    if (attn) attn += u * T * d;
    alpha += u * gate_ld;
    eta += u * gate_ld;
    theta += u * gate_ld;
    const int nch = (int)((T + chunk - 1) / chunk);
    const int c1 = min(nch, (s + 1) * G);
    for (int c = s * G; c < c1; ++c) {
        const long t0 = (long)c * chunk;
        const int n = (int)min((long)chunk, T - t0);
        chunk_scan(alpha, eta, theta, t0, n, chunk, chunk_gates, s_a, s_e, s_t, s_c, s_d, s_scal);
        const float An = s_scal[0], En = s_scal[1], sig = s_scal[2];
        const Tin* K = k + t0 * d;
        const Tin* Q = q + t0 * d;
        const Tin* V = v + t0 * d;
        for (int idx = tid; idx < n * d; idx += blockDim.x) {  // G = 2 (W k - v), y = W q
            const int t = idx / d, i = idx % d;
            float yh = 0.f, yq = 0.f;
            const float* Wr = X + (size_t)i * d2;
            for (int m = 0; m < d; ++m) {
                yh += Wr[m] * ldx(K + (size_t)t * d + m);
                yq += Wr[m] * ldx(Q + (size_t)t * d + m);
            }
            Ge[idx] = 2.f * (yh - ldx(V + idx));
            const long o = (t0 + t) * d + i;
            stx(y + o, attn ? ldx(attn + o) / (1.f + expf(-yq)) : yq);
        }
        __syncthreads();
        for (int idx = tid; idx < d * d; idx += blockDim.x) {
            const int i = idx / d, m = idx % d;
            float uc = 0.f, ud = 0.f;
            for (int t = 0; t < n; ++t) {
                const float g = Ge[(size_t)t * d + i] * ldx(K + (size_t)t * d + m);
                uc += s_c[t] * g;
                ud += s_d[t] * g;
            }
            float* Wr = X + (size_t)i * d2;
            const float w = Wr[m], sv = Wr[d + m];
            Wr[m] = An * w + sig * sv - uc;
            Wr[d + m] = En * sv - ud;
        }
        __syncthreads();
    }
    if (s == nseg_used - 1) {
        for (int idx = tid; idx < d * d; idx += blockDim.x) {
            const int i = idx / d, m = idx % d;
            Wout[u * d * d + idx] = X[(size_t)i * d2 + m];
            Sout[u * d * d + idx] = X[(size_t)i * d2 + d + m];
        }
    }
}

// 3'. The same run with the state, the chunk's keys and queries and G in shared memory (d = 64,
// chunks up to 64 tokens): X [d][2d], K and Q [n][d + 1] (one padding column), G [d][n].
__host__ __device__ inline size_t run_smem_bytes(int chunk) {
    constexpr int d = 64;
    return ((size_t)2 * d * d + (size_t)2 * chunk * (d + 1) + (size_t)chunk * d) * sizeof(float);
}

template <typename Tin>
__global__ void __launch_bounds__(kScanThreads) linear_scan_run_smem(
    long T, long gate_ld, int chunk, int chunk_gates, int nseg_used, int G, const Tin* __restrict__ k,
    const Tin* __restrict__ q, const Tin* __restrict__ v, const float* __restrict__ alpha,
    const float* __restrict__ eta, const float* __restrict__ theta, float* __restrict__ Wout,
    float* __restrict__ Sout, Tin* __restrict__ y, const Tin* __restrict__ attn, float* __restrict__ ws,
    size_t ws_per_unit) {
    constexpr int d = 64, d2 = 128;
    __shared__ float s_a[kScanMaxChunk], s_e[kScanMaxChunk], s_t[kScanMaxChunk], s_c[kScanMaxChunk],
        s_d[kScanMaxChunk], s_scal[3];
    extern __shared__ float smf[];
    float* sX = smf;                          // [d][2d]: W | S
    float* sK = sX + d * d2;                  // [n][d + 1]
    float* sQ = sK + (size_t)chunk * (d + 1);
    float* sG = sQ + (size_t)chunk * (d + 1);  // [d][n]
    const long u = blockIdx.x / nseg_used;
    const int s = blockIdx.x % nseg_used, tid = threadIdx.x;
    const float* X0 = ws + u * ws_per_unit + (size_t)s * slot_floats(d, chunk) + (size_t)6 * d * d +
                      (size_t)3 * d * chunk;
    for (int i = tid; i < d * d2 / 4; i += blockDim.x)
        reinterpret_cast<float4*>(sX)[i] = reinterpret_cast<const float4*>(X0)[i];
    k += u * T * d;
    q += u * T * d;
    v += u * T * d;
    y += u * T * d;
    if (attn) attn += u * T * d;
    alpha += u * gate_ld;
    eta += u * gate_ld;
    theta += u * gate_ld;
    const int nch = (int)((T + chunk - 1) / chunk);
    const int c1 = min(nch, (s + 1) * G);
    for (int c = s * G; c < c1; ++c) {
        const long t0 = (long)c * chunk;
        const int n = (int)min((long)chunk, T - t0);
        chunk_scan(alpha, eta, theta, t0, n, chunk, chunk_gates, s_a, s_e, s_t, s_c, s_d, s_scal);
        const float An = s_scal[0], En = s_scal[1], sig = s_scal[2];
        for (int idx = tid; idx < n * d; idx += blockDim.x) {
            const int t = idx / d, m = idx % d;
            sK[t * (d + 1) + m] = ldx(k + t0 * d + idx);
            sQ[t * (d + 1) + m] = ldx(q + t0 * d + idx);
        }
        __syncthreads();
        // G = 2 (W k - v), y = W q; the lanes of a warp take consecutive tokens of one output row i,
        // so the row of W is a broadcast and the key rows (padded) hit distinct banks. G is [d][n].
        for (int idx = tid; idx < n * d; idx += blockDim.x) {
            const int i = idx / n, t = idx % n;
            float yh = 0.f, yq = 0.f;
            const float* Wr = sX + i * d2;
            const float* Kt = sK + t * (d + 1);
            const float* Qt = sQ + t * (d + 1);
#pragma unroll 8
            for (int m = 0; m < d; ++m) {
                yh = fmaf(Wr[m], Kt[m], yh);
                yq = fmaf(Wr[m], Qt[m], yq);
            }
            const long o = (t0 + t) * d + i;
            sG[i * n + t] = 2.f * (yh - ldx(v + o));
            stx(y + o, attn ? ldx(attn + o) / (1.f + expf(-yq)) : yq);
        }
        __syncthreads();
        for (int idx = tid; idx < d * d; idx += blockDim.x) {
            const int i = idx / d, m = idx % d;
            float uc = 0.f, ud = 0.f;
            for (int t = 0; t < n; ++t) {
                const float g = sG[i * n + t] * sK[t * (d + 1) + m];
                uc = fmaf(s_c[t], g, uc);
                ud = fmaf(s_d[t], g, ud);
            }
            float* Wr = sX + i * d2;
            const float w = Wr[m], sv = Wr[d + m];
            Wr[m] = An * w + sig * sv - uc;
            Wr[d + m] = En * sv - ud;
        }
        __syncthreads();
    }
    if (s == nseg_used - 1) {
        for (int idx = tid; idx < d * d; idx += blockDim.x) {
            const int i = idx / d, m = idx % d;
            Wout[u * d * d + idx] = sX[i * d2 + m];
            Sout[u * d * d + idx] = sX[i * d2 + d + m];
        }
    }
}

template <typename Tin>
static cudaError_t launch_scan(const ForwardArgs& a, int nseg_max, cudaStream_t st) {
    const int nch = (int)((a.T + a.chunk - 1) / a.chunk);
    int nseg = nseg_max < 1 ? 1 : nseg_max;
    if (nseg > nch) nseg = nch;
    const int G = (nch + nseg - 1) / nseg;
    const int used = (nch + G - 1) / G;  // segments that hold chunks
    const unsigned grid = (unsigned)(a.units * used);
    cudaError_t e = cudaSuccess;
    if (a.d == kSegSmemD && a.chunk <= kComposeSmemMaxChunk) {
        static std::atomic<unsigned> attr_set{0};  // per device: set before the first launch there
        int dev = 0;
        e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= 32) return cudaErrorInvalidDevice;
        if (!(attr_set.load() & (1u << dev))) {
            e = cudaFuncSetAttribute(linear_scan_compose_smem<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)compose_smem_bytes(kComposeSmemMaxChunk));
            if (e != cudaSuccess) return e;
            attr_set.fetch_or(1u << dev);
        }
        linear_scan_compose_smem<Tin><<<grid, kScanThreads, compose_smem_bytes(a.chunk), st>>>(
            a.T, a.gate_ld, a.chunk, (int)a.chunk_gates, used, G, (const Tin*)a.k, (const Tin*)a.v, a.alpha, a.eta,
            a.theta, a.ws, a.ws_per_unit);
    } else {
        linear_scan_compose<Tin><<<grid, kScanThreads, 0, st>>>(a.d, a.T, a.gate_ld, a.chunk, (int)a.chunk_gates,
                                                                used, G, (const Tin*)a.k, (const Tin*)a.v, a.alpha,
                                                                a.eta, a.theta, a.ws, a.ws_per_unit);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (a.d == kSegSmemD) {
        static std::atomic<unsigned> attr_set{0};  // per device: set before the first launch there
        int dev = 0;
        e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= 32) return cudaErrorInvalidDevice;
        if (!(attr_set.load() & (1u << dev))) {
            e = cudaFuncSetAttribute(linear_scan_segments_smem, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kSegSmemBytes);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(linear_scan_tree_level, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kTreeSmemBytes);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(linear_scan_tree_apply, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kTreeSmemBytes);
            if (e != cudaSuccess) return e;
            attr_set.fetch_or(1u << dev);
        }
        if (used >= kTreeMinSegments) {
            // tree over the segments: ceil(log2 used) composition levels, then every start state at once
            int src2 = 0;
            for (int step = 1; step < used; step <<= 1) {
                linear_scan_tree_level<<<grid, kScanThreads, kTreeSmemBytes, st>>>(a.chunk, used, step, src2, a.ws,
                                                                                   a.ws_per_unit);
                e = cudaGetLastError();
                if (e != cudaSuccess) return e;
                src2 ^= 1;
            }
            linear_scan_tree_apply<<<grid, kScanThreads, kTreeSmemBytes, st>>>(a.chunk, used, src2, a.W1, a.S1, a.ws,
                                                                               a.ws_per_unit);
        } else {
            linear_scan_segments_smem<<<(unsigned)a.units, kScanThreads, kSegSmemBytes, st>>>(a.chunk, used, a.W1,
                                                                                               a.S1, a.ws,
                                                                                               a.ws_per_unit);
        }
    } else {
        linear_scan_segments<<<(unsigned)a.units, kScanThreads, 0, st>>>(a.d, a.chunk, used, used, a.W1, a.S1, a.ws,
                                                                         a.ws_per_unit);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (a.d == kSegSmemD && a.chunk <= kComposeSmemMaxChunk) {
        static std::atomic<unsigned> attr_set{0};  // per device: set before the first launch there
        int dev = 0;
        e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= 32) return cudaErrorInvalidDevice;
        if (!(attr_set.load() & (1u << dev))) {
            e = cudaFuncSetAttribute(linear_scan_run_smem<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)run_smem_bytes(kComposeSmemMaxChunk));
            if (e != cudaSuccess) return e;
            attr_set.fetch_or(1u << dev);
        }
        linear_scan_run_smem<Tin><<<grid, kScanThreads, run_smem_bytes(a.chunk), st>>>(
            a.T, a.gate_ld, a.chunk, (int)a.chunk_gates, used, G, (const Tin*)a.k, (const Tin*)a.q, (const Tin*)a.v,
            a.alpha, a.eta, a.theta, a.W1, a.S1, (Tin*)a.y, (const Tin*)a.attn, a.ws, a.ws_per_unit);
    } else {
        linear_scan_run<Tin><<<grid, kScanThreads, 0, st>>>(a.d, a.T, a.gate_ld, a.chunk, (int)a.chunk_gates, used,
                                                            G, (const Tin*)a.k, (const Tin*)a.q, (const Tin*)a.v,
                                                            a.alpha, a.eta, a.theta, a.W1, a.S1, (Tin*)a.y,
                                                            (const Tin*)a.attn, a.ws, a.ws_per_unit);
    }
    return cudaGetLastError();
}

cudaError_t launch_linear_scan(const ForwardArgs& a, int nseg_max, cudaStream_t st) {
    if (a.h != 0 || a.chunk > kScanMaxChunk) return cudaErrorInvalidValue;
    return a.bf16 ? launch_scan<__nv_bfloat16>(a, nseg_max, st) : launch_scan<float>(a, nseg_max, st);
}

}  // namespace titans
