// CUDA-core (SIMT) chunk kernel: fp32 reference mode of the memory's chunk-wise
// forward, for the linear and the MLP memory at any supported shape.
//
// Follows the tensorized mini-batch form of "Titans: Learning to Memorize at Test
// Time" (walk-through sec. 3.2): every token of a chunk takes its gradient at the
// chunk-start weights, so the chunk's n momentum/forgetting steps (sec. 3.1) fold
// into per-token coefficients and three per-chunk scalars:
//   W_end = A W_0 + sigma S_0 - sum_j c_j g_j,   S_end = E S_0 - sum_j d_j g_j,
//   P_j = prod_{l>j} (1 - alpha_l), Q_j = prod_{l>j} eta_l,
//   r_{n-1} = 1, r_j = P_j + eta_{j+1} r_{j+1}, c_j = theta_j r_j, d_j = theta_j Q_j,
//   A = (1 - alpha_0) P_0, E = eta_0 Q_0, sigma = eta_0 r_0.
// One CTA per unit; intermediates of a chunk live in the handle's workspace
// (global memory, L2-resident), the state in the caller's buffers.
#include <cuda_bf16.h>
#include <cstdint>

#include "kernels.h"

namespace titans {

__device__ __forceinline__ float ldin(const float* p) { return *p; }
__device__ __forceinline__ float ldin(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void stout(float* p, float v) { *p = v; }
__device__ __forceinline__ void stout(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// The retrieval M(q) itself, or the memory-as-a-gate output attn * sigmoid(M(q)) ("Titans",
// walk-through sec. 4.2 "Gated Memory": the logistic function of the memory's retrieval gates
// the attention branch's output element-wise).
template <typename Tin>
__device__ __forceinline__ float gated(float yq, const Tin* attn, long idx) {
    return attn ? ldin(attn + idx) * (1.f / (1.f + expf(-yq))) : yq;
}

constexpr int kCcThreads = 1024;
constexpr int kCcMaxChunk = 128;

// Workspace floats per unit for chunk length n (MLP: Zk, Ak, Aq, Dl [n][h] and G [n][d];
// linear: G [n][d]).
__host__ size_t cuda_cores_ws_floats(int d, int h, int n) {
    return h ? (size_t)4 * n * h + (size_t)n * d : (size_t)n * d;
}

template <typename Tin>
__global__ void __launch_bounds__(kCcThreads) chunk_fwd_cuda_cores(
    int d, int h, long T, long gate_ld, int chunk, int chunk_gates, const Tin* __restrict__ k, const Tin* __restrict__ q,
    const Tin* __restrict__ v, const float* __restrict__ alpha, const float* __restrict__ eta,
    const float* __restrict__ theta, float* __restrict__ W1, float* __restrict__ W2, float* __restrict__ S1,
    float* __restrict__ S2, Tin* __restrict__ y, const Tin* __restrict__ attn, float* __restrict__ ws,
    size_t ws_per_unit) {
    __shared__ float s_alpha[kCcMaxChunk], s_eta[kCcMaxChunk], s_theta[kCcMaxChunk];
    __shared__ float s_c[kCcMaxChunk], s_d[kCcMaxChunk], s_scal[3];

    const int tid = threadIdx.x;
    const long u = blockIdx.x;
    const size_t nW1 = h ? (size_t)h * d : (size_t)d * d;
    const size_t nW2 = (size_t)d * h;
    k += u * T * d;
    q += u * T * d;
    v += u * T * d;
    y += u * T * d;
    if (attn) attn += u * T * d;
    alpha += u * gate_ld;
    eta += u * gate_ld;
    theta += u * gate_ld;
    W1 += u * nW1;
    S1 += u * nW1;
    if (h) {
        W2 += u * nW2;
        S2 += u * nW2;
    }
    float* wsu = ws + u * ws_per_unit;
    float* Zk = wsu;                         // [n][h] keys' pre-activations
    float* Ak = Zk + (size_t)chunk * h;      // [n][h] silu(Zk)
    float* Aq = Ak + (size_t)chunk * h;      // [n][h] silu(queries' pre-activations)
    float* Dl = Aq + (size_t)chunk * h;      // [n][h] backprop to W1
    float* G = h ? Dl + (size_t)chunk * h : wsu;  // [n][d] 2 (M(k) - v)

    for (long t0 = 0; t0 < T; t0 += chunk) {
        const int n = (int)min((long)chunk, T - t0);
        for (int i = tid; i < n; i += blockDim.x) {
            const long gi = chunk_gates ? t0 / chunk : t0 + i;  // chunk-shared or per-token gates
            s_alpha[i] = alpha[gi];
            s_eta[i] = eta[gi];
            s_theta[i] = theta[gi];
        }
        __syncthreads();
        if (tid == 0) {  // suffix scan, division-free
            float Pr = 1.f, Qr = 1.f, r_next = 0.f;
            for (int j = n - 1; j >= 0; --j) {
                const float r = Pr + (j + 1 < n ? s_eta[j + 1] * r_next : 0.f);
                s_c[j] = s_theta[j] * r;
                s_d[j] = s_theta[j] * Qr;
                r_next = r;
                Pr *= 1.f - s_alpha[j];
                Qr *= s_eta[j];
            }
            s_scal[0] = Pr;                // A = prod (1 - alpha)
            s_scal[1] = Qr;                // E = prod eta
            s_scal[2] = s_eta[0] * r_next; // sigma = eta_0 r_0
        }
        __syncthreads();
        const float An = s_scal[0], En = s_scal[1], sig = s_scal[2];
        const Tin* K = k + t0 * d;
        const Tin* Q = q + t0 * d;
        const Tin* V = v + t0 * d;

        if (h == 0) {  // linear memory M(x) = W x
            for (int idx = tid; idx < n * d; idx += blockDim.x) {
                const int t = idx / d, i = idx % d;
                float yh = 0.f, yq = 0.f;
                for (int m = 0; m < d; ++m) {
                    const float w = W1[(size_t)i * d + m];
                    yh += w * ldin(K + (size_t)t * d + m);
                    yq += w * ldin(Q + (size_t)t * d + m);
                }
                G[idx] = 2.f * (yh - ldin(V + idx));
                stout(y + (t0 + t) * d + i, gated(yq, attn, (t0 + t) * d + i));
            }
            __syncthreads();
            for (int idx = tid; idx < d * d; idx += blockDim.x) {
                const int i = idx / d, m = idx % d;
                float uc = 0.f, ud = 0.f;
                for (int t = 0; t < n; ++t) {
                    const float g = G[(size_t)t * d + i] * ldin(K + (size_t)t * d + m);
                    uc += s_c[t] * g;
                    ud += s_d[t] * g;
                }
                const float w = W1[idx], s = S1[idx];
                W1[idx] = An * w + sig * s - uc;
                S1[idx] = En * s - ud;
            }
            __syncthreads();
            continue;
        }

        // MLP memory M(x) = W2 silu(W1 x)
        for (int idx = tid; idx < n * h; idx += blockDim.x) {
            const int t = idx / h, j = idx % h;
            float z = 0.f, zq = 0.f;
            for (int m = 0; m < d; ++m) {
                const float w = W1[(size_t)j * d + m];
                z += w * ldin(K + (size_t)t * d + m);
                zq += w * ldin(Q + (size_t)t * d + m);
            }
            Zk[idx] = z;
            Ak[idx] = z / (1.f + expf(-z));
            Aq[idx] = zq / (1.f + expf(-zq));
        }
        __syncthreads();
        for (int idx = tid; idx < n * d; idx += blockDim.x) {
            const int t = idx / d, i = idx % d;
            float yh = 0.f, yq = 0.f;
            for (int j = 0; j < h; ++j) {
                const float w = W2[(size_t)i * h + j];
                yh += w * Ak[(size_t)t * h + j];
                yq += w * Aq[(size_t)t * h + j];
            }
            G[idx] = 2.f * (yh - ldin(V + idx));
            stout(y + (t0 + t) * d + i, gated(yq, attn, (t0 + t) * d + i));
        }
        __syncthreads();
        for (int idx = tid; idx < n * h; idx += blockDim.x) {
            const int t = idx / h, j = idx % h;
            float b = 0.f;
            for (int i = 0; i < d; ++i) b += W2[(size_t)i * h + j] * G[(size_t)t * d + i];
            const float z = Zk[idx];
            const float s = 1.f / (1.f + expf(-z));
            Dl[idx] = b * s * (1.f + z * (1.f - s));
        }
        __syncthreads();
        for (int idx = tid; idx < d * h; idx += blockDim.x) {  // W2, S2 [d][h]
            const int i = idx / h, j = idx % h;
            float uc = 0.f, ud = 0.f;
            for (int t = 0; t < n; ++t) {
                const float g = G[(size_t)t * d + i] * Ak[(size_t)t * h + j];
                uc += s_c[t] * g;
                ud += s_d[t] * g;
            }
            const float w = W2[idx], s = S2[idx];
            W2[idx] = An * w + sig * s - uc;
            S2[idx] = En * s - ud;
        }
        for (int idx = tid; idx < h * d; idx += blockDim.x) {  // W1, S1 [h][d]
            const int j = idx / d, m = idx % d;
            float uc = 0.f, ud = 0.f;
            for (int t = 0; t < n; ++t) {
                const float g = Dl[(size_t)t * h + j] * ldin(K + (size_t)t * d + m);
                uc += s_c[t] * g;
                ud += s_d[t] * g;
            }
            const float w = W1[idx], s = S1[idx];
            W1[idx] = An * w + sig * s - uc;
            S1[idx] = En * s - ud;
        }
        __syncthreads();
    }
}

template <typename Tin>
cudaError_t launch_cuda_cores(const ForwardArgs& a, cudaStream_t st) {
    chunk_fwd_cuda_cores<Tin><<<(unsigned)a.units, kCcThreads, 0, st>>>(
        a.d, a.h, a.T, a.gate_ld, a.chunk, (int)a.chunk_gates, (const Tin*)a.k, (const Tin*)a.q, (const Tin*)a.v, a.alpha, a.eta, a.theta, a.W1,
        a.W2, a.S1, a.S2, (Tin*)a.y, (const Tin*)a.attn, a.ws, a.ws_per_unit);
    return cudaGetLastError();
}

cudaError_t launch_chunk_cuda_cores(const ForwardArgs& a, cudaStream_t st) {
    return a.bf16 ? launch_cuda_cores<__nv_bfloat16>(a, st) : launch_cuda_cores<float>(a, st);
}

// Querying a kernel's attributes makes the runtime load its code on the current device, so
// that no later launch has to (under lazy module loading the first launch would otherwise).
cudaError_t preload_chunk_cuda_cores() {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, chunk_fwd_cuda_cores<float>);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, chunk_fwd_cuda_cores<__nv_bfloat16>);
    return e;
}

}  // namespace titans
