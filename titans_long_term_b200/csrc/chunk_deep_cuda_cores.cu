// CUDA-core chunk kernel of the deep memory M(x) = W_L silu(W_{L-1} ... silu(W_1 x)), L >= 2
// layers, every hidden layer h wide, no bias ("Titans: Learning to Memorize at Test Time",
// walk-through sec. 3.1 "Memory Architecture": an MLP with L_M >= 2 layers; sec. 5.5 "The Effect
// of Deep Memory"). fp32 arithmetic; k, q, v, y in fp32 or bf16.
//
// Per chunk (every token's gradient at the chunk-start weights, sec. 3.2), one CTA per unit:
//   gate scan -> c_j, d_j, A, E, sigma (division-free suffix scan, as in the 2-layer kernels);
//   keys forward through every layer, keeping each hidden layer's pre-activation and activation;
//   queries forward through the same chunk-start layers -> y (or the gated output);
//   delta = 2 (M(k) - v), then from the output layer down: the next delta
//   (W_l^T delta) * silu'(z_{l-1}) is taken with the chunk-start W_l, and only then is layer l
//   updated, W_l <- A W_l + sigma S_l - sum_j c_j delta_j in_j^T, S_l <- E S_l - sum_j d_j ...
// The state is packed per unit, layers one after another, each row-major [out][in]:
// W_1 [h][d], W_2 .. W_{L-1} [h][h], W_L [d][h].
#include <cuda_bf16.h>
#include <cstdint>

#include "kernels.h"

namespace titans {

namespace {

__device__ __forceinline__ float ld_in(const float* p) { return *p; }
__device__ __forceinline__ float ld_in(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_out(float* p, float v) { *p = v; }
__device__ __forceinline__ void st_out(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

constexpr int kDeepThreads = 1024;
constexpr int kDeepMaxChunk = 128;

__device__ __forceinline__ float sigm(float z) { return 1.f / (1.f + expf(-z)); }

__host__ __device__ __forceinline__ size_t layer_offset(int d, int h, int l) {
    return l == 0 ? 0 : (size_t)h * d + (size_t)(l - 1) * h * h;
}

// out[t][o] = sum_m W[o][m] in[t][m] for t < n (one output element per thread-iteration);
// with act: a[t][o] = silu(out[t][o]) too.
template <typename Tin>
__device__ void dense(int n, int n_out, int n_in, const float* W, const Tin* in_tok, const float* in_act,
                      float* z, float* act) {
    for (int idx = threadIdx.x; idx < n * n_out; idx += blockDim.x) {
        const int t = idx / n_out, o = idx % n_out;
        float s = 0.f;
        const float* w = W + (size_t)o * n_in;
        if (in_act) {
            const float* x = in_act + (size_t)t * n_in;
            for (int m = 0; m < n_in; ++m) s += w[m] * x[m];
        } else {
            const Tin* x = in_tok + (size_t)t * n_in;
            for (int m = 0; m < n_in; ++m) s += w[m] * ld_in(x + m);
        }
        z[idx] = s;
        if (act) act[idx] = s * sigm(s);
    }
}

}  // namespace

// Workspace floats per unit: keys' pre-activations and activations of the L-1 hidden layers,
// two query-activation buffers, two delta buffers (each [n][h]) and the output error [n][d].
size_t deep_ws_floats(int d, int h, int layers, int n) {
    return (size_t)2 * (layers - 1) * n * h + (size_t)4 * n * h + (size_t)n * d;
}

__host__ __device__ size_t deep_state_floats(int d, int h, int layers) {
    return (size_t)2 * h * d + (size_t)(layers - 2) * h * h;
}

template <typename Tin>
__global__ void __launch_bounds__(kDeepThreads) chunk_fwd_deep_cuda_cores(
    int d, int h, int L, long T, long gate_ld, int chunk, int chunk_gates, const Tin* __restrict__ k, const Tin* __restrict__ q,
    const Tin* __restrict__ v, const float* __restrict__ alpha, const float* __restrict__ eta,
    const float* __restrict__ theta, float* __restrict__ W, float* __restrict__ S, Tin* __restrict__ y,
    const Tin* __restrict__ attn, float* __restrict__ ws, size_t ws_per_unit) {
    __shared__ float s_alpha[kDeepMaxChunk], s_eta[kDeepMaxChunk], s_theta[kDeepMaxChunk];
    __shared__ float s_c[kDeepMaxChunk], s_d[kDeepMaxChunk], s_scal[3];
    const int tid = threadIdx.x;
    const long u = blockIdx.x;
    const size_t P = deep_state_floats(d, h, L);
    k += u * T * d;
    q += u * T * d;
    v += u * T * d;
    y += u * T * d;
    if (attn) attn += u * T * d;
    alpha += u * gate_ld;
    eta += u * gate_ld;
    theta += u * gate_ld;
    W += u * P;
    S += u * P;
    float* wsu = ws + u * ws_per_unit;
    const size_t nh = (size_t)chunk * h;
    float* Zk = wsu;                          // [L-1][n][h] keys' pre-activations
    float* Ak = Zk + (size_t)(L - 1) * nh;    // [L-1][n][h] keys' activations
    float* Qa = Ak + (size_t)(L - 1) * nh;    // [2][n][h]   queries' activations (ping-pong)
    float* Dl = Qa + 2 * nh;                  // [2][n][h]   delta (ping-pong)
    float* Ge = Dl + 2 * nh;                  // [n][d]      2 (M(k) - v), the output layer's delta

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
            s_scal[0] = Pr;
            s_scal[1] = Qr;
            s_scal[2] = s_eta[0] * r_next;
        }
        __syncthreads();
        const float An = s_scal[0], En = s_scal[1], sig = s_scal[2];
        const Tin* K = k + t0 * d;
        const Tin* Q = q + t0 * d;
        const Tin* V = v + t0 * d;

        // Keys forward through the hidden layers.
        for (int l = 0; l < L - 1; ++l) {
            const float* Wl = W + layer_offset(d, h, l);
            dense<Tin>(n, h, l == 0 ? d : h, Wl, K, l == 0 ? nullptr : Ak + (size_t)(l - 1) * nh, Zk + (size_t)l * nh,
                       Ak + (size_t)l * nh);
            __syncthreads();
        }
        // Queries forward through the same chunk-start layers (activations only, two buffers in turn).
        for (int l = 0; l < L - 1; ++l) {
            const float* Wl = W + layer_offset(d, h, l);
            float* outa = Qa + (size_t)(l & 1) * nh;
            dense<Tin>(n, h, l == 0 ? d : h, Wl, Q, l == 0 ? nullptr : Qa + (size_t)((l - 1) & 1) * nh, outa, outa);
            __syncthreads();
        }
        {
            const float* WL = W + layer_offset(d, h, L - 1);
            const float* ak = Ak + (size_t)(L - 2) * nh;
            const float* aq = Qa + (size_t)((L - 2) & 1) * nh;
            for (int idx = tid; idx < n * d; idx += blockDim.x) {
                const int t = idx / d, i = idx % d;
                float yh = 0.f, yq = 0.f;
                const float* w = WL + (size_t)i * h;
                for (int j = 0; j < h; ++j) {
                    yh += w[j] * ak[(size_t)t * h + j];
                    yq += w[j] * aq[(size_t)t * h + j];
                }
                Ge[idx] = 2.f * (yh - ld_in(V + idx));
                const long o = (t0 + t) * d + i;
                st_out(y + o, attn ? ld_in(attn + o) * sigm(yq) : yq);
            }
        }
        __syncthreads();

        // Backward from the output layer; each layer is updated once its delta has gone through it.
        const float* delta = Ge;
        int n_out = d;
        for (int l = L - 1; l >= 0; --l) {
            float* Wl = W + layer_offset(d, h, l);
            float* Sl = S + layer_offset(d, h, l);
            const int n_in = l == 0 ? d : h;
            float* next = Dl + (size_t)(l & 1) * nh;
            if (l > 0) {  // next delta with the chunk-start W_l: (W_l^T delta) * silu'(z_{l-1})
                const float* zp = Zk + (size_t)(l - 1) * nh;
                for (int idx = tid; idx < n * h; idx += blockDim.x) {
                    const int t = idx / h, m = idx % h;
                    float b = 0.f;
                    for (int o = 0; o < n_out; ++o) b += Wl[(size_t)o * h + m] * delta[(size_t)t * n_out + o];
                    const float z = zp[idx], sg = sigm(z);
                    next[idx] = b * sg * (1.f + z * (1.f - sg));
                }
                __syncthreads();
            }
            // W_l <- A W_l + sigma S_l - sum_j c_j delta_j in_j^T;  S_l <- E S_l - sum_j d_j delta_j in_j^T
            const float* in_act = l == 0 ? nullptr : Ak + (size_t)(l - 1) * nh;
            for (int idx = tid; idx < n_out * n_in; idx += blockDim.x) {
                const int o = idx / n_in, m = idx % n_in;
                float uc = 0.f, ud = 0.f;
                for (int t = 0; t < n; ++t) {
                    const float x = in_act ? in_act[(size_t)t * h + m] : ld_in(K + (size_t)t * d + m);
                    const float g = delta[(size_t)t * n_out + o] * x;
                    uc += s_c[t] * g;
                    ud += s_d[t] * g;
                }
                const float w = Wl[idx], s = Sl[idx];
                Wl[idx] = An * w + sig * s - uc;
                Sl[idx] = En * s - ud;
            }
            __syncthreads();
            delta = next;
            n_out = h;
        }
    }
}

template <typename Tin>
static cudaError_t launch_deep(const ForwardArgs& a, int layers, cudaStream_t st) {
    chunk_fwd_deep_cuda_cores<Tin><<<(unsigned)a.units, kDeepThreads, 0, st>>>(
        a.d, a.h, layers, a.T, a.gate_ld, a.chunk, (int)a.chunk_gates, (const Tin*)a.k, (const Tin*)a.q, (const Tin*)a.v, a.alpha, a.eta,
        a.theta, a.W1, a.S1, (Tin*)a.y, (const Tin*)a.attn, a.ws, a.ws_per_unit);
    return cudaGetLastError();
}

cudaError_t launch_chunk_deep_cuda_cores(const ForwardArgs& a, int layers, cudaStream_t st) {
    if (a.chunk > kDeepMaxChunk || layers < 2) return cudaErrorInvalidValue;
    return a.bf16 ? launch_deep<__nv_bfloat16>(a, layers, st) : launch_deep<float>(a, layers, st);
}

}  // namespace titans
