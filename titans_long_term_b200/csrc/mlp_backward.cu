// Backward of the chunked 2-layer MLP memory M(x) = W2 silu(W1 x): gradients of
// L = <dy, y> + <dW1, W1_T> + <dW2, W2_T> + <dS1, S1_T> + <dS2, S2_T> with respect to k, q, v, the
// gates and the initial W1, W2, S1, S2 ("Titans: Learning to Memorize at Test Time": the forward of
// walk-through sec. 3.1-3.2; k, v, q come from the outer loop's projections).
//
// One chunk (tokens j, chunk-start W1 [h][d], W2 [d][h], S1, S2; c_j, d_j, A, E, sigma from the gate
// scan), forward:
//   z_j = W1 k_j, a_j = silu(z_j), g_j = 2 (W2 a_j - v_j), b_j = W2^T g_j, delta_j = b_j * silu'(z_j),
//   zq_j = W1 q_j, y_j = W2 silu(zq_j),
//   W2' = A W2 + sigma S2 - sum c_j g_j a_j^T,   S2' = E S2 - sum d_j g_j a_j^T,
//   W1' = A W1 + sigma S1 - sum c_j delta_j k_j^T, S1' = E S1 - sum d_j delta_j k_j^T.
// Adjoint, given the chunk-end adjoints dW1', dW2', dS1', dS2' and dy_j:
//   dg_j = -(c_j dW2' + d_j dS2') a_j,  da_j = -(c_j dW2'^T + d_j dS2'^T) g_j,
//   ddelta_j = -(c_j dW1' + d_j dS1') k_j,  dk_j = -(c_j dW1'^T + d_j dS1'^T) delta_j,
//   dc_j = -g_j . dW2' a_j - delta_j . dW1' k_j,  dd_j = the same with dS2', dS1';
//   db_j = ddelta_j * silu'(z_j),  dz_j = ddelta_j * b_j * silu''(z_j);
//   dg_j += W2 db_j,  dW2 += g_j db_j^T;  dyhat_j = 2 dg_j, dv_j = -2 dg_j;
//   da_j += W2^T dyhat_j,  dW2 += dyhat_j a_j^T;  dz_j += da_j * silu'(z_j);
//   dk_j += W1^T dz_j,  dW1 += dz_j k_j^T;
//   queries: dzq_j = (W2^T dy_j) * silu'(zq_j), dW2 += dy_j silu(zq_j)^T, dW1 += dzq_j q_j^T, dq_j = W1^T dzq_j;
//   dW1 += A dW1', dW2 += A dW2', dS1 = sigma dW1' + E dS1', dS2 = sigma dW2' + E dS2',
//   dA = <dW1', W1> + <dW2', W2>, dsigma = <dW1', S1> + <dW2', S2>, dE = <dS1', S1> + <dS2', S2>,
// and the gates back through the scan as in the linear memory's backward (division-free).
// silu'(z) = s (1 + z (1 - s)), silu''(z) = s (1 - s) (2 + z (1 - 2 s)), s = sigmoid(z).
// Pass 1 reruns the forward keeping every chunk-start state in the caller's workspace; pass 2
// walks the chunks backwards. One CTA per unit, fp32 on CUDA cores.
#include <cuda_bf16.h>
#include <cstdint>

#include "kernels.h"

namespace titans {

namespace {

__device__ __forceinline__ float ldm(const float* p) { return *p; }
__device__ __forceinline__ float ldm(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void stm(float* p, float v) { *p = v; }
__device__ __forceinline__ void stm(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
__device__ __forceinline__ float sgm(float z) { return 1.f / (1.f + expf(-z)); }

constexpr int kMbThreads = 1024;
constexpr int kMbMaxChunk = 128;

}  // namespace

// Workspace floats per unit: every chunk-start state (4 h d each), two adjoint sets (2 x 4 h d), and
// per-chunk activations: Z, A, B, Delta, dA, dZ, Zq, Aq ([n][h] each), G, dG ([n][d]), and the terms of
// dc_j, dd_j ([2][n][d + h]).
size_t mlp_backward_ws_floats(int d, int h, long T, int chunk) {
    const long nch = (T + chunk - 1) / chunk;
    return (size_t)nch * 4 * h * d + (size_t)8 * h * d + (size_t)8 * chunk * h + (size_t)2 * chunk * d +
           (size_t)2 * chunk * (d + h);
}

template <typename Tin>
__global__ void __launch_bounds__(kMbThreads) mlp_backward_kernel(MlpBackwardArgs a) {
    __shared__ float s_a[kMbMaxChunk], s_e[kMbMaxChunk], s_t[kMbMaxChunk];
    __shared__ float s_c[kMbMaxChunk], s_d[kMbMaxChunk], s_r[kMbMaxChunk], s_P[kMbMaxChunk], s_Q[kMbMaxChunk];
    __shared__ float s_dc[kMbMaxChunk], s_dd[kMbMaxChunk], s_scal[3], s_red[3];
    const int tid = threadIdx.x, d = a.d, h = a.h, chunk = a.chunk;
    const long u = blockIdx.x, T = a.T;
    const long nch = (T + chunk - 1) / chunk;
    const size_t hd = (size_t)h * d, nh = (size_t)chunk * h;
    const Tin* k = (const Tin*)a.k + (size_t)u * T * d;
    const Tin* q = (const Tin*)a.q + (size_t)u * T * d;
    const Tin* v = (const Tin*)a.v + (size_t)u * T * d;
    const Tin* dy = (const Tin*)a.dy + (size_t)u * T * d;
    Tin* dk = (Tin*)a.dk + (size_t)u * T * d;
    Tin* dq = (Tin*)a.dq + (size_t)u * T * d;
    Tin* dv = (Tin*)a.dv + (size_t)u * T * d;
    const float* alpha = a.alpha + (size_t)u * T;
    const float* eta = a.eta + (size_t)u * T;
    const float* theta = a.theta + (size_t)u * T;
    float* dalpha = a.dalpha + (size_t)u * T;
    float* deta = a.deta + (size_t)u * T;
    float* dtheta = a.dtheta + (size_t)u * T;
    float* ws = a.ws + u * a.ws_per_unit;
    float* Xs = ws;                                   // [nch][W1 | W2 | S1 | S2], 4 h d each
    float* dX = Xs + (size_t)nch * 4 * hd;            // [2][4 h d] adjoints (chunk end, chunk start)
    float* Zb = dX + (size_t)8 * hd;                  // [n][h]
    float* Ab = Zb + nh;
    float* Bb = Ab + nh;
    float* Dl = Bb + nh;                              // delta
    float* dAb = Dl + nh;
    float* dZb = dAb + nh;
    float* Zq = dZb + nh;
    float* Aq = Zq + nh;
    float* Gb = Aq + nh;                              // [n][d]
    float* dGb = Gb + (size_t)chunk * d;
    float* Tc = dGb + (size_t)chunk * d;              // terms of dc_j, dd_j: [n][d + h] each
    float* Td = Tc + (size_t)chunk * (d + h);

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
    // Keys' and queries' forward at the state X (W1 at X, W2 at X + hd): Z, A, G, B, Delta, Zq, Aq.
    auto forward = [&](const float* X, long t0, int n, bool queries) {
        const float* W1 = X;
        const float* W2 = X + hd;
        for (int idx = tid; idx < n * h; idx += blockDim.x) {
            const int t = idx / h, j = idx % h;
            float z = 0.f, zq = 0.f;
            for (int m = 0; m < d; ++m) {
                const float w = W1[(size_t)j * d + m];
                z += w * ldm(k + (t0 + t) * d + m);
                if (queries) zq += w * ldm(q + (t0 + t) * d + m);
            }
            Zb[idx] = z;
            Ab[idx] = z * sgm(z);
            if (queries) {
                Zq[idx] = zq;
                Aq[idx] = zq * sgm(zq);
            }
        }
        __syncthreads();
        for (int idx = tid; idx < n * d; idx += blockDim.x) {
            const int t = idx / d, i = idx % d;
            float yh = 0.f;
            for (int j = 0; j < h; ++j) yh += W2[(size_t)i * h + j] * Ab[(size_t)t * h + j];
            Gb[idx] = 2.f * (yh - ldm(v + (t0 + t) * d + i));
        }
        __syncthreads();
        for (int idx = tid; idx < n * h; idx += blockDim.x) {
            const int t = idx / h, j = idx % h;
            float b = 0.f;
            for (int i = 0; i < d; ++i) b += W2[(size_t)i * h + j] * Gb[(size_t)t * d + i];
            const float z = Zb[idx], s = sgm(z);
            Bb[idx] = b;
            Dl[idx] = b * s * (1.f + z * (1.f - s));
        }
        __syncthreads();
    };

    // ---- pass 1: the forward, keeping each chunk-start state
    for (size_t i = tid; i < 4 * hd; i += blockDim.x) {
        const float* src = i < hd ? a.W1 : (i < 2 * hd ? a.W2 : (i < 3 * hd ? a.S1 : a.S2));
        Xs[i] = src[u * hd + (i % hd)];
    }
    __syncthreads();
    for (long c = 0; c + 1 < nch; ++c) {
        const long t0 = c * chunk;
        const int n = (int)min((long)chunk, T - t0);
        scan(t0, n);
        const float An = s_scal[0], En = s_scal[1], sig = s_scal[2];
        const float* X = Xs + (size_t)c * 4 * hd;
        float* Xn = Xs + (size_t)(c + 1) * 4 * hd;
        forward(X, t0, n, false);
        for (int idx = tid; idx < d * h; idx += blockDim.x) {  // W2, S2 [d][h]
            const int i = idx / h, j = idx % h;
            float uc = 0.f, ud = 0.f;
            for (int t = 0; t < n; ++t) {
                const float g = Gb[(size_t)t * d + i] * Ab[(size_t)t * h + j];
                uc += s_c[t] * g;
                ud += s_d[t] * g;
            }
            Xn[hd + idx] = An * X[hd + idx] + sig * X[3 * hd + idx] - uc;
            Xn[3 * hd + idx] = En * X[3 * hd + idx] - ud;
        }
        for (int idx = tid; idx < h * d; idx += blockDim.x) {  // W1, S1 [h][d]
            const int j = idx / d, m = idx % d;
            float uc = 0.f, ud = 0.f;
            for (int t = 0; t < n; ++t) {
                const float g = Dl[(size_t)t * h + j] * ldm(k + (t0 + t) * d + m);
                uc += s_c[t] * g;
                ud += s_d[t] * g;
            }
            Xn[idx] = An * X[idx] + sig * X[2 * hd + idx] - uc;
            Xn[2 * hd + idx] = En * X[2 * hd + idx] - ud;
        }
        __syncthreads();
    }

    // ---- pass 2: backwards
    float* dcur = dX;             // adjoint at the chunk's end: dW1', dW2', dS1', dS2'
    float* dnext = dX + 4 * hd;   // adjoint at its start
    for (size_t i = tid; i < 4 * hd; i += blockDim.x) {
        const float* src = i < hd ? a.dW1 : (i < 2 * hd ? a.dW2 : (i < 3 * hd ? a.dS1 : a.dS2));
        dcur[i] = src ? src[u * hd + (i % hd)] : 0.f;
    }
    __syncthreads();
    for (long c = nch - 1; c >= 0; --c) {
        const long t0 = c * chunk;
        const int n = (int)min((long)chunk, T - t0);
        scan(t0, n);
        const float An = s_scal[0], En = s_scal[1], sig = s_scal[2];
        const float* X = Xs + (size_t)c * 4 * hd;
        const float* W1 = X;
        const float* W2 = X + hd;
        const float* dW1e = dcur;
        const float* dW2e = dcur + hd;
        const float* dS1e = dcur + 2 * hd;
        const float* dS2e = dcur + 3 * hd;
        forward(X, t0, n, true);
        if (tid < 3) s_red[tid] = 0.f;
        // chunk scalars' adjoints
        {
            float pa = 0.f, ps = 0.f, pe = 0.f;
            for (size_t i = tid; i < 2 * hd; i += blockDim.x) {
                pa += dcur[i] * X[i];
                ps += dcur[i] * X[2 * hd + i];
                pe += dcur[2 * hd + i] * X[2 * hd + i];
            }
            __syncthreads();
            atomicAdd(&s_red[0], pa);
            atomicAdd(&s_red[1], ps);
            atomicAdd(&s_red[2], pe);
        }
        // dg_j = -(c_j dW2' + d_j dS2') a_j   [n][d]
        for (int idx = tid; idx < n * d; idx += blockDim.x) {
            const int t = idx / d, i = idx % d;
            float x2 = 0.f, y2 = 0.f;
            for (int j = 0; j < h; ++j) {
                const float aj = Ab[(size_t)t * h + j];
                x2 += dW2e[(size_t)i * h + j] * aj;
                y2 += dS2e[(size_t)i * h + j] * aj;
            }
            dGb[idx] = -(s_c[t] * x2 + s_d[t] * y2);
            // dc_j, dd_j terms -g_j . dW2' a_j, -g_j . dS2' a_j (summed per token below)
            const float g = Gb[idx];
            Tc[(size_t)t * (d + h) + i] = -g * x2;
            Td[(size_t)t * (d + h) + i] = -g * y2;
        }
        // da_j = -(c_j dW2'^T + d_j dS2'^T) g_j;  ddelta_j = -(c_j dW1' + d_j dS1') k_j   [n][h]
        for (int idx = tid; idx < n * h; idx += blockDim.x) {
            const int t = idx / h, j = idx % h;
            float x2 = 0.f, y2 = 0.f, x1 = 0.f, y1 = 0.f;
            for (int i = 0; i < d; ++i) {
                const float g = Gb[(size_t)t * d + i];
                x2 += dW2e[(size_t)i * h + j] * g;
                y2 += dS2e[(size_t)i * h + j] * g;
            }
            for (int m = 0; m < d; ++m) {
                const float km = ldm(k + (t0 + t) * d + m);
                x1 += dW1e[(size_t)j * d + m] * km;
                y1 += dS1e[(size_t)j * d + m] * km;
            }
            dAb[idx] = -(s_c[t] * x2 + s_d[t] * y2);
            const float ddel = -(s_c[t] * x1 + s_d[t] * y1);
            // dc_j, dd_j terms -delta_j . dW1' k_j, -delta_j . dS1' k_j
            Tc[(size_t)t * (d + h) + d + j] = -Dl[idx] * x1;
            Td[(size_t)t * (d + h) + d + j] = -Dl[idx] * y1;
            // db = ddelta * silu'(z); dz = ddelta * b * silu''(z)
            const float z = Zb[idx], s = sgm(z);
            dZb[idx] = ddel * Bb[idx] * s * (1.f - s) * (2.f + z * (1.f - 2.f * s));
            Bb[idx] = ddel * s * (1.f + z * (1.f - s));  // Bb now holds db
        }
        __syncthreads();
        // dc_j, dd_j: one warp per token sums its d + h terms in a fixed order (lane-strided, then
        // a shuffle tree), so the result does not depend on scheduling.
        for (int t = tid >> 5; t < n; t += blockDim.x >> 5) {
            const int lane = tid & 31;
            float sc = 0.f, sd = 0.f;
            for (int i = lane; i < d + h; i += 32) {
                sc += Tc[(size_t)t * (d + h) + i];
                sd += Td[(size_t)t * (d + h) + i];
            }
            for (int off = 16; off > 0; off >>= 1) {
                sc += __shfl_xor_sync(0xffffffffu, sc, off);
                sd += __shfl_xor_sync(0xffffffffu, sd, off);
            }
            if (lane == 0) {
                s_dc[t] = sc;
                s_dd[t] = sd;
            }
        }
        // dg_j += W2 db_j;  then dyhat = 2 dg, dv = -2 dg
        for (int idx = tid; idx < n * d; idx += blockDim.x) {
            const int t = idx / d, i = idx % d;
            float s = 0.f;
            for (int j = 0; j < h; ++j) s += W2[(size_t)i * h + j] * Bb[(size_t)t * h + j];
            const float g = dGb[idx] + s;
            dGb[idx] = 2.f * g;  // dyhat
            stm(dv + (t0 + t) * d + i, -2.f * g);
        }
        __syncthreads();
        // da_j += W2^T dyhat_j;  dz_j += da_j * silu'(z_j)
        for (int idx = tid; idx < n * h; idx += blockDim.x) {
            const int t = idx / h, j = idx % h;
            float s = 0.f;
            for (int i = 0; i < d; ++i) s += W2[(size_t)i * h + j] * dGb[(size_t)t * d + i];
            const float da = dAb[idx] + s;
            const float z = Zb[idx], sg = sgm(z);
            dZb[idx] += da * sg * (1.f + z * (1.f - sg));
        }
        // queries: dzq_j = (W2^T dy_j) * silu'(zq_j) (into Zq)
        for (int idx = tid; idx < n * h; idx += blockDim.x) {
            const int t = idx / h, j = idx % h;
            float s = 0.f;
            for (int i = 0; i < d; ++i) s += W2[(size_t)i * h + j] * ldm(dy + (t0 + t) * d + i);
            const float z = Zq[idx], sg = sgm(z);
            Zq[idx] = s * sg * (1.f + z * (1.f - sg));
        }
        __syncthreads();
        // dk_j = -(c_j dW1'^T + d_j dS1'^T) delta_j + W1^T dz_j;  dq_j = W1^T dzq_j
        for (int idx = tid; idx < n * d; idx += blockDim.x) {
            const int t = idx / d, m = idx % d;
            float x1 = 0.f, y1 = 0.f, wz = 0.f, wq = 0.f;
            for (int j = 0; j < h; ++j) {
                const float dl = Dl[(size_t)t * h + j];
                x1 += dW1e[(size_t)j * d + m] * dl;
                y1 += dS1e[(size_t)j * d + m] * dl;
                wz += W1[(size_t)j * d + m] * dZb[(size_t)t * h + j];
                wq += W1[(size_t)j * d + m] * Zq[(size_t)t * h + j];
            }
            stm(dk + (t0 + t) * d + m, -(s_c[t] * x1 + s_d[t] * y1) + wz);
            stm(dq + (t0 + t) * d + m, wq);
        }
        // chunk-start adjoints
        for (int idx = tid; idx < h * d; idx += blockDim.x) {  // dW1 [h][d], dS1
            const int j = idx / d, m = idx % d;
            float acc = An * dW1e[idx];
            for (int t = 0; t < n; ++t)
                acc += dZb[(size_t)t * h + j] * ldm(k + (t0 + t) * d + m) + Zq[(size_t)t * h + j] * ldm(q + (t0 + t) * d + m);
            dnext[idx] = acc;
            dnext[2 * hd + idx] = sig * dW1e[idx] + En * dS1e[idx];
        }
        for (int idx = tid; idx < d * h; idx += blockDim.x) {  // dW2 [d][h], dS2
            const int i = idx / h, j = idx % h;
            float acc = An * dW2e[idx];
            for (int t = 0; t < n; ++t) {
                const float g = Gb[(size_t)t * d + i];
                // g_j db_j^T + dyhat_j a_j^T + dy_j aq_j^T
                acc += g * Bb[(size_t)t * h + j] + dGb[(size_t)t * d + i] * Ab[(size_t)t * h + j] +
                       ldm(dy + (t0 + t) * d + i) * Aq[(size_t)t * h + j];
            }
            dnext[hd + idx] = acc;
            dnext[3 * hd + idx] = sig * dW2e[idx] + En * dS2e[idx];
        }
        __syncthreads();
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
    for (size_t i = tid; i < 4 * hd; i += blockDim.x) {
        float* dst = i < hd ? a.dW1_0 : (i < 2 * hd ? a.dW2_0 : (i < 3 * hd ? a.dS1_0 : a.dS2_0));
        dst[u * hd + (i % hd)] = dcur[i];
    }
}

cudaError_t launch_mlp_backward(const MlpBackwardArgs& a, cudaStream_t st) {
    if (a.chunk < 1 || a.chunk > kMbMaxChunk) return cudaErrorInvalidValue;
    if (a.bf16)
        mlp_backward_kernel<__nv_bfloat16><<<(unsigned)a.units, kMbThreads, 0, st>>>(a);
    else
        mlp_backward_kernel<float><<<(unsigned)a.units, kMbThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace titans
