// Backward of the chunked linear memory M(x) = W x: gradients of a scalar loss
// L = <dy, y> + <dW_T, W_T> + <dS_T, S_T> with respect to k, q, v, alpha, eta, theta and the initial
// W, S ("Titans: Learning to Memorize at Test Time": the memory's forward of walk-through sec. 3.1-
// 3.2; its inputs k, v, q come from outer-loop projections W_K, W_V, W_Q that training learns).
//
// One chunk (tokens j = 0..n-1, chunk-start W, S; c_j, d_j, A, E, sigma from the gate scan):
//   y_j = W q_j,   e_j = W k_j - v_j,
//   W' = A W + sigma S - 2 sum_j c_j e_j k_j^T,   S' = E S - 2 sum_j d_j e_j k_j^T.
// Its adjoint, given dW', dS' and dy_j:
//   dE_j = -2 (c_j dW' k_j + d_j dS' k_j),     dv_j = -dE_j,     dq_j = W^T dy_j,
//   dk_j = -2 (c_j dW'^T e_j + d_j dS'^T e_j) + W^T dE_j,
//   dc_j = -2 e_j . (dW' k_j),   dd_j = -2 e_j . (dS' k_j),
//   dA = <dW', W>,  dsigma = <dW', S>,  dE = <dS', S>,
//   dW = A dW' + sum_j dE_j k_j^T + sum_j dy_j q_j^T,   dS = sigma dW' + E dS'.
// The gates' adjoints go back through the scan P_j = prod_{l>j} (1 - alpha_l), Q_j = prod_{l>j} eta_l,
// r_j = P_j + eta_{j+1} r_{j+1}, c_j = theta_j r_j, d_j = theta_j Q_j, A = (1 - alpha_0) P_0,
// E = eta_0 Q_0, sigma = eta_0 r_0, without divisions:
//   dtheta_j = dc_j r_j + dd_j Q_j;   dr_j = theta_j dc_j + eta_j dr_{j-1} (+ eta_0 dsigma at j = 0);
//   dalpha_l = -P_l F_l with F_0 = dA, F_{l+1} = (1 - alpha_l) F_l + dr_l;
//   deta_l = Q_l H_l + (l > 0 ? dr_{l-1} r_l : dsigma r_0) with H_0 = dE, H_{l+1} = eta_l H_l + theta_l dd_l.
// A first pass reruns the forward and keeps every chunk-start state in the caller's workspace; the
// second pass walks the chunks backwards. One CTA per unit, fp32 on CUDA cores.
#include <cuda_bf16.h>
#include <cstdint>

#include "kernels.h"

namespace titans {

namespace {

__device__ __forceinline__ float ldb(const float* p) { return *p; }
__device__ __forceinline__ float ldb(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void stb(float* p, float v) { *p = v; }
__device__ __forceinline__ void stb(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

constexpr int kBwdThreads = 256;
constexpr int kBwdMaxChunk = 128;

}  // namespace

// Workspace floats per unit: every chunk-start state [W | S] (2 d^2 each), two adjoint buffers
// [d][2d], and e_j, dW' k_j, dS' k_j, dE_j ([n][d] each).
size_t linear_backward_ws_floats(int d, long T, int chunk) {
    const long nch = (T + chunk - 1) / chunk;
    return (size_t)nch * 2 * d * d + (size_t)4 * d * d + (size_t)4 * chunk * d;
}

template <typename Tin>
__global__ void __launch_bounds__(kBwdThreads) linear_backward_kernel(
    int d, long T, int chunk, const Tin* __restrict__ k, const Tin* __restrict__ q, const Tin* __restrict__ v,
    const float* __restrict__ alpha, const float* __restrict__ eta, const float* __restrict__ theta,
    const float* __restrict__ W0, const float* __restrict__ S0, const Tin* __restrict__ dy,
    const float* __restrict__ dWT, const float* __restrict__ dST, Tin* __restrict__ dk, Tin* __restrict__ dq,
    Tin* __restrict__ dv, float* __restrict__ dalpha, float* __restrict__ deta, float* __restrict__ dtheta,
    float* __restrict__ dW0, float* __restrict__ dS0, float* __restrict__ ws, size_t ws_per_unit) {
    __shared__ float s_a[kBwdMaxChunk], s_e[kBwdMaxChunk], s_t[kBwdMaxChunk];
    __shared__ float s_c[kBwdMaxChunk], s_d[kBwdMaxChunk], s_r[kBwdMaxChunk], s_P[kBwdMaxChunk], s_Q[kBwdMaxChunk];
    __shared__ float s_dc[kBwdMaxChunk], s_dd[kBwdMaxChunk], s_scal[3], s_red[3];
    const int tid = threadIdx.x;
    const long u = blockIdx.x;
    const int d2 = 2 * d;
    const long nch = (T + chunk - 1) / chunk;
    const size_t off_tok = (size_t)u * T * d, off_g = (size_t)u * T, off_w = (size_t)u * d * d;
    float* Xs = ws + u * ws_per_unit;               // [nch][d][2d] chunk-start states
    float* dX = Xs + (size_t)nch * 2 * d * d;       // [2][d][2d] adjoint buffers
    float* Eb = dX + (size_t)4 * d * d;             // [n][d] e_j
    float* Ub = Eb + (size_t)chunk * d;             // [n][d] dW' k_j
    float* Vb = Ub + (size_t)chunk * d;             // [n][d] dS' k_j
    float* Db = Vb + (size_t)chunk * d;             // [n][d] dE_j
    k += off_tok;
    q += off_tok;
    v += off_tok;
    dy += off_tok;
    dk += off_tok;
    dq += off_tok;
    dv += off_tok;
    alpha += off_g;
    eta += off_g;
    theta += off_g;
    dalpha += off_g;
    deta += off_g;
    dtheta += off_g;

    // Gate scan of chunk c into shared memory (also keeps r_j, P_j, Q_j for the adjoint).
    auto scan = [&](long t0, int n) {
        for (int i = tid; i < n; i += blockDim.x) {
            s_a[i] = alpha[t0 + i];
            s_e[i] = eta[t0 + i];
            s_t[i] = theta[t0 + i];
        }
        __syncthreads();
        if (tid == 0) {
            float Pr = 1.f, Qr = 1.f, r_next = 0.f;
            for (int j = n - 1; j >= 0; --j) {
                const float r = Pr + (j + 1 < n ? s_e[j + 1] * r_next : 0.f);
                s_r[j] = r;
                s_P[j] = Pr;
                s_Q[j] = Qr;
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
    };

    // ---- pass 1: the forward, keeping each chunk-start state
    for (int idx = tid; idx < d * d2; idx += blockDim.x) {
        const int i = idx / d2, j = idx % d2;
        Xs[idx] = j < d ? W0[off_w + (size_t)i * d + j] : S0[off_w + (size_t)i * d + (j - d)];
    }
    __syncthreads();
    for (long c = 0; c + 1 < nch; ++c) {
        const long t0 = c * chunk;
        const int n = (int)min((long)chunk, T - t0);
        scan(t0, n);
        const float An = s_scal[0], En = s_scal[1], sig = s_scal[2];
        const float* X = Xs + (size_t)c * d * d2;
        float* Xn = Xs + (size_t)(c + 1) * d * d2;
        for (int idx = tid; idx < n * d; idx += blockDim.x) {  // e_j
            const int t = idx / d, i = idx % d;
            float s = 0.f;
            for (int m = 0; m < d; ++m) s += X[(size_t)i * d2 + m] * ldb(k + (t0 + t) * d + m);
            Eb[idx] = s - ldb(v + (t0 + t) * d + i);
        }
        __syncthreads();
        for (int idx = tid; idx < d * d; idx += blockDim.x) {
            const int i = idx / d, m = idx % d;
            float uc = 0.f, ud = 0.f;
            for (int t = 0; t < n; ++t) {
                const float g = Eb[(size_t)t * d + i] * ldb(k + (t0 + t) * d + m);
                uc += s_c[t] * g;
                ud += s_d[t] * g;
            }
            const float w = X[(size_t)i * d2 + m], s = X[(size_t)i * d2 + d + m];
            Xn[(size_t)i * d2 + m] = An * w + sig * s - 2.f * uc;
            Xn[(size_t)i * d2 + d + m] = En * s - 2.f * ud;
        }
        __syncthreads();
    }

    // ---- pass 2: backwards through the chunks
    float* dcur = dX;                      // adjoint of the state after the current chunk
    float* dnext = dX + (size_t)2 * d * d;  // adjoint of its chunk-start state
    for (int idx = tid; idx < d * d2; idx += blockDim.x) {
        const int i = idx / d2, j = idx % d2;
        const float* src = j < d ? dWT : dST;
        dcur[idx] = src ? src[off_w + (size_t)i * d + (j < d ? j : j - d)] : 0.f;
    }
    __syncthreads();
    for (long c = nch - 1; c >= 0; --c) {
        const long t0 = c * chunk;
        const int n = (int)min((long)chunk, T - t0);
        scan(t0, n);
        const float An = s_scal[0], En = s_scal[1], sig = s_scal[2];
        const float* X = Xs + (size_t)c * d * d2;
        if (tid < 3) s_red[tid] = 0.f;
        // e_j = W k_j - v_j, dW' k_j, dS' k_j
        for (int idx = tid; idx < n * d; idx += blockDim.x) {
            const int t = idx / d, i = idx % d;
            float e = 0.f, uw = 0.f, us = 0.f;
            for (int m = 0; m < d; ++m) {
                const float km = ldb(k + (t0 + t) * d + m);
                e += X[(size_t)i * d2 + m] * km;
                uw += dcur[(size_t)i * d2 + m] * km;
                us += dcur[(size_t)i * d2 + d + m] * km;
            }
            Eb[idx] = e - ldb(v + (t0 + t) * d + i);
            Ub[idx] = uw;
            Vb[idx] = us;
        }
        __syncthreads();
        // per token: dc_j, dd_j and dE_j; the chunk scalars' adjoints
        for (int t = tid; t < n; t += blockDim.x) {
            float sc = 0.f, sd = 0.f;
            for (int i = 0; i < d; ++i) {
                sc += Eb[(size_t)t * d + i] * Ub[(size_t)t * d + i];
                sd += Eb[(size_t)t * d + i] * Vb[(size_t)t * d + i];
            }
            s_dc[t] = -2.f * sc;
            s_dd[t] = -2.f * sd;
        }
        for (int idx = tid; idx < n * d; idx += blockDim.x) {
            const int t = idx / d;
            Db[idx] = -2.f * (s_c[t] * Ub[idx] + s_d[t] * Vb[idx]);
        }
        {
            float pa = 0.f, ps = 0.f, pe = 0.f;
            for (int idx = tid; idx < d * d; idx += blockDim.x) {
                const int i = idx / d, m = idx % d;
                const float gw = dcur[(size_t)i * d2 + m], gs = dcur[(size_t)i * d2 + d + m];
                pa += gw * X[(size_t)i * d2 + m];
                ps += gw * X[(size_t)i * d2 + d + m];
                pe += gs * X[(size_t)i * d2 + d + m];
            }
            atomicAdd(&s_red[0], pa);
            atomicAdd(&s_red[1], ps);
            atomicAdd(&s_red[2], pe);
        }
        __syncthreads();
        // dk, dv, dq of the chunk's tokens
        for (int idx = tid; idx < n * d; idx += blockDim.x) {
            const int t = idx / d, m = idx % d;
            float a = 0.f, b = 0.f, wde = 0.f, wdy = 0.f;
            for (int i = 0; i < d; ++i) {
                const float e = Eb[(size_t)t * d + i];
                a += dcur[(size_t)i * d2 + m] * e;
                b += dcur[(size_t)i * d2 + d + m] * e;
                const float wim = X[(size_t)i * d2 + m];
                wde += wim * Db[(size_t)t * d + i];
                wdy += wim * ldb(dy + (t0 + t) * d + i);
            }
            stb(dk + (t0 + t) * d + m, -2.f * (s_c[t] * a + s_d[t] * b) + wde);
            stb(dq + (t0 + t) * d + m, wdy);
            stb(dv + (t0 + t) * d + m, -Db[(size_t)t * d + m]);
        }
        // adjoint of the chunk-start state
        for (int idx = tid; idx < d * d; idx += blockDim.x) {
            const int i = idx / d, m = idx % d;
            float acc = An * dcur[(size_t)i * d2 + m];
            for (int t = 0; t < n; ++t)
                acc += Db[(size_t)t * d + i] * ldb(k + (t0 + t) * d + m) +
                       ldb(dy + (t0 + t) * d + i) * ldb(q + (t0 + t) * d + m);
            dnext[(size_t)i * d2 + m] = acc;
            dnext[(size_t)i * d2 + d + m] = sig * dcur[(size_t)i * d2 + m] + En * dcur[(size_t)i * d2 + d + m];
        }
        // the gates, back through the scan
        if (tid == 0) {
            const float dA = s_red[0], dsig = s_red[1], dE = s_red[2];
            float dr_prev = 0.f, F = dA, H = dE;
            for (int j = 0; j < n; ++j) {
                const float dr = s_t[j] * s_dc[j] + (j == 0 ? s_e[0] * dsig : s_e[j] * dr_prev);
                dtheta[t0 + j] = s_dc[j] * s_r[j] + s_dd[j] * s_Q[j];
                dalpha[t0 + j] = -s_P[j] * F;
                deta[t0 + j] = s_Q[j] * H + (j == 0 ? dsig * s_r[0] : dr_prev * s_r[j]);
                F = (1.f - s_a[j]) * F + dr;
                H = s_e[j] * H + s_t[j] * s_dd[j];
                dr_prev = dr;
            }
        }
        __syncthreads();
        float* tmp = dcur;
        dcur = dnext;
        dnext = tmp;
    }
    for (int idx = tid; idx < d * d; idx += blockDim.x) {
        const int i = idx / d, m = idx % d;
        dW0[off_w + idx] = dcur[(size_t)i * d2 + m];
        dS0[off_w + idx] = dcur[(size_t)i * d2 + d + m];
    }
}

cudaError_t launch_linear_backward(const LinearBackwardArgs& b, cudaStream_t st) {
    if (b.chunk < 1 || b.chunk > kBwdMaxChunk) return cudaErrorInvalidValue;
    if (b.bf16)
        linear_backward_kernel<__nv_bfloat16><<<(unsigned)b.units, kBwdThreads, 0, st>>>(
            b.d, b.T, b.chunk, (const __nv_bfloat16*)b.k, (const __nv_bfloat16*)b.q, (const __nv_bfloat16*)b.v,
            b.alpha, b.eta, b.theta, b.W0, b.S0, (const __nv_bfloat16*)b.dy, b.dWT, b.dST, (__nv_bfloat16*)b.dk,
            (__nv_bfloat16*)b.dq, (__nv_bfloat16*)b.dv, b.dalpha, b.deta, b.dtheta, b.dW0, b.dS0, b.ws,
            b.ws_per_unit);
    else
        linear_backward_kernel<float><<<(unsigned)b.units, kBwdThreads, 0, st>>>(
            b.d, b.T, b.chunk, (const float*)b.k, (const float*)b.q, (const float*)b.v, b.alpha, b.eta, b.theta,
            b.W0, b.S0, (const float*)b.dy, b.dWT, b.dST, (float*)b.dk, (float*)b.dq, (float*)b.dv, b.dalpha,
            b.deta, b.dtheta, b.dW0, b.dS0, b.ws, b.ws_per_unit);
    return cudaGetLastError();
}

}  // namespace titans
