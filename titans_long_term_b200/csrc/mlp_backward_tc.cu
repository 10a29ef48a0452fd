// Backward of the chunked 2-layer MLP memory M(x) = W2 silu(W1 x) on tensor cores (d = 64,
// h = 256, chunk <= 64, bf16 token streams): the gradients of
// L = <dy, y> + <dW1, W1_T> + <dW2, W2_T> + <dS1, S1_T> + <dS2, S2_T> with respect to k, q, v, the
// gates and the initial W1, W2, S1, S2, as the CUDA-core backward computes them ("Titans: Learning
// to Memorize at Test Time", walk-through sec. 3.1-3.2 for the forward; k, v, q come from the outer
// loop's projections).
//
// One CTA per unit, 8 warps, 512 TMEM columns. Every per-chunk product is a 128-row tcgen05 GEMM
// with bf16 operands in shared memory and an fp32 accumulator in TMEM; each of the 128 TMEM lanes
// is one thread's row in the epilogue. A chunk's keys fill rows 0..63 of a tile and its queries
// rows 64..127, so that the key and query halves of a step share one MMA group:
//   Z = [K; Q] W1^T;  Y = [A_q; A] W2^T (keys' rows 64..127);  [G; dy] W2 = [B; W2^T dy]
// and the outer-product sums over a chunk's tokens stack their factors along K:
//   dW1 += [dz; dzq]^T [K; Q],   dW2^T += [db; A_q; A]^T [G; dy; dyhat].
// The c- and d-weighted adjoint products fold the two weights into one K-stacked operand:
//   [c G | d G] [dW2'; dS2'] and [c K | d K] [dW1' | dS1']^T.
// Pass 1 runs the chunk forward (the same GEMMs plus the weighted outer products) and keeps every
// chunk-start state; pass 2 walks the chunks backwards. The chunk scalars' adjoints and the gates'
// adjoints through the division-free scan follow the CUDA-core backward.
#include <cuda_bf16.h>

#include <atomic>
#include <cstdint>

#include "kernels.h"
#include "phased_common.cuh"
#include "ptx.cuh"

namespace titans {

namespace mbt {
constexpr int kD = 64, kH = 256, kN = 64, kThreads = 256;
constexpr size_t kHD = (size_t)kH * kD;
constexpr uint32_t kBOff = 64 * 1024;  // B operand tiles (A at 0)
constexpr uint32_t kOperands = 192 * 1024;
constexpr uint32_t SCAN = kOperands;           // alpha, eta, theta, c, d, r, P, Q [8][64] floats
constexpr uint32_t DCS = SCAN + 8 * 64 * 4;    // dc, dd [2][64]
constexpr uint32_t PART = DCS + 2 * 64 * 4;    // half-row partials [2][2][128]
constexpr uint32_t RED = PART + 4 * 128 * 4;   // per-warp partial dots [8][4]
constexpr uint32_t SCAL = RED + 8 * 4 * 4;     // A, E, sigma
constexpr uint32_t BAR = SCAL + 16 * 4;
constexpr uint32_t TPTR = BAR + 8;
constexpr uint32_t END = TPTR + 8;
constexpr size_t kSmemBytes = END + 1024;
constexpr uint32_t kTmemCols = 512;

// Byte offsets of a unit's workspace pieces.
struct Layout {
    size_t ckpt, adj, w1b, w2b, dw1b, dw2b, xq, ck, pq, gq, cg, dz, dl, sp, spp, spq, bm, da0, dz0, gf, dg0, total;
};
__host__ __device__ inline size_t a1k(size_t x) { return (x + 1023) & ~size_t(1023); }
__host__ __device__ inline Layout layout(long nch) {
    Layout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = a1k(o + bytes);
        return at;
    };
    L.ckpt = take((size_t)nch * 4 * kHD * 4);  // fp32 chunk-start states [nch][W1 | W2 | S1 | S2]
    L.adj = take(4 * kHD * 4);                 // fp32 adjoint, updated in place chunk by chunk
    L.w1b = take(kHD * 2);                     // bf16 W1 [h][d]
    L.w2b = take(kHD * 2);                     // bf16 W2 [d][h]
    L.dw1b = take(kHD * 2 * 2);                // bf16 [h][dW1' | dS1']
    L.dw2b = take(kHD * 2 * 2);                // bf16 [dW2'; dS2'] [2d][h]
    L.xq = take((size_t)128 * kD * 2);         // bf16 [K; Q]
    L.ck = take((size_t)128 * 2 * kD * 2);     // bf16 [c K | d K]
    L.pq = take((size_t)256 * kH * 2);         // bf16 [db; A_q; A; 0]
    L.gq = take((size_t)256 * kD * 2);         // bf16 [G; dy; dyhat; 0]
    L.cg = take((size_t)128 * 2 * kD * 2);     // bf16 [c G | d G]
    L.dz = take((size_t)128 * kH * 2);         // bf16 [dz; dzq]
    L.dl = take((size_t)128 * kH * 2);         // bf16 [Delta; 0]
    L.sp = take((size_t)kN * kH * 4);          // fp32 silu'(Z_K)
    L.spp = take((size_t)kN * kH * 4);         // fp32 silu''(Z_K)
    L.spq = take((size_t)kN * kH * 4);         // fp32 silu'(Z_Q)
    L.bm = take((size_t)kN * kH * 4);          // fp32 B = G W2
    L.da0 = take((size_t)kN * kH * 4);         // fp32 dA from the W2 update terms
    L.dz0 = take((size_t)kN * kH * 4);         // fp32 dz from the W1 update terms
    L.gf = take((size_t)kN * kD * 4);          // fp32 G
    L.dg0 = take((size_t)kN * kD * 4);         // fp32 dG from the W2 update terms
    L.total = o;
    return L;
}
}  // namespace mbt

namespace {

using phc::cp_async16;
using phc::cp_async_wait_all;
using phc::load_kmajor;
using phc::load_mnmajor;
using phc::mma_steps;
using phc::operands_ready;
using phc::pack2;
using phc::tanh_approx;

__device__ __forceinline__ void st16_bf16(__nv_bfloat16* dst, const float (&x)[16]) {
    uint4* p = reinterpret_cast<uint4*>(dst);
    p[0] = make_uint4(pack2(x[0], x[1]), pack2(x[2], x[3]), pack2(x[4], x[5]), pack2(x[6], x[7]));
    p[1] = make_uint4(pack2(x[8], x[9]), pack2(x[10], x[11]), pack2(x[12], x[13]), pack2(x[14], x[15]));
}
__device__ __forceinline__ void ld16_bf16(const __nv_bfloat16* src, float (&x)[16]) {
    const uint4* p = reinterpret_cast<const uint4*>(src);
    const uint4 a = p[0], b = p[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 f = unpack_bf16x2(w[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}
// fp32 per-token scratch is stored token-contiguous ([column][64 tokens]) so that the 32 lanes of a
// warp, one token row each, read and write 128 contiguous bytes per column.
__device__ __forceinline__ void ldcol16(const float* base, int col, int t, float (&x)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) x[e] = base[(size_t)(col + e) * 64 + t];
}
__device__ __forceinline__ void stcol16(float* base, int col, int t, const float (&x)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) base[(size_t)(col + e) * 64 + t] = x[e];
}
__device__ __forceinline__ void tmem16(uint32_t taddr, float (&x)[16]) {
    uint32_t r[16];
    tmem_ld16(taddr, r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = __uint_as_float(r[i]);
}

}  // namespace

__global__ void __launch_bounds__(mbt::kThreads, 1) mlp_backward_tc_kernel(const __grid_constant__ MlpBackwardArgs a) {
    using namespace mbt;
    using bf16 = __nv_bfloat16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + BAR);
    float* s_a = reinterpret_cast<float*>(sm + SCAN);
    float* s_e = s_a + 64;
    float* s_t = s_a + 128;
    float* s_c = s_a + 192;
    float* s_d = s_a + 256;
    float* s_r = s_a + 320;
    float* s_P = s_a + 384;
    float* s_Q = s_a + 448;
    float* s_dc = reinterpret_cast<float*>(sm + DCS);
    float* s_dd = s_dc + 64;
    float* s_part = reinterpret_cast<float*>(sm + PART);  // [c|d][half][row]
    float* s_red = reinterpret_cast<float*>(sm + RED);
    float* s_scal = reinterpret_cast<float*>(sm + SCAL);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    const int row = 32 * quad + lane;  // this thread's TMEM lane = tile row

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(reinterpret_cast<uint32_t*>(sm + TPTR), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + TPTR);
    uint32_t mma_phase = 0;
    bool ok = true;
#define DBG(cond) TITANS_DBG(cond, a.status, static_cast<volatile int*>(nullptr))

    const long u = blockIdx.x, T = a.T;
    const int chunk = a.chunk;
    const long nch = (T + chunk - 1) / chunk;
    const Layout Lw = layout(nch);
    uint8_t* ws = reinterpret_cast<uint8_t*>(a.ws) + (size_t)u * a.ws_per_unit * sizeof(float);
    float* ckpt = reinterpret_cast<float*>(ws + Lw.ckpt);
    float* adj = reinterpret_cast<float*>(ws + Lw.adj);
    bf16* W1b = reinterpret_cast<bf16*>(ws + Lw.w1b);
    bf16* W2b = reinterpret_cast<bf16*>(ws + Lw.w2b);
    bf16* dW1b = reinterpret_cast<bf16*>(ws + Lw.dw1b);
    bf16* dW2b = reinterpret_cast<bf16*>(ws + Lw.dw2b);
    bf16* XQ = reinterpret_cast<bf16*>(ws + Lw.xq);
    bf16* CK = reinterpret_cast<bf16*>(ws + Lw.ck);
    bf16* PQ = reinterpret_cast<bf16*>(ws + Lw.pq);
    bf16* GQ = reinterpret_cast<bf16*>(ws + Lw.gq);
    bf16* CG = reinterpret_cast<bf16*>(ws + Lw.cg);
    bf16* DZ = reinterpret_cast<bf16*>(ws + Lw.dz);
    bf16* DL = reinterpret_cast<bf16*>(ws + Lw.dl);
    float* SP = reinterpret_cast<float*>(ws + Lw.sp);
    float* SPP = reinterpret_cast<float*>(ws + Lw.spp);
    float* SPQ = reinterpret_cast<float*>(ws + Lw.spq);
    float* BM = reinterpret_cast<float*>(ws + Lw.bm);
    float* DA0 = reinterpret_cast<float*>(ws + Lw.da0);
    float* DZ0 = reinterpret_cast<float*>(ws + Lw.dz0);
    float* GF = reinterpret_cast<float*>(ws + Lw.gf);
    float* DG0 = reinterpret_cast<float*>(ws + Lw.dg0);
    const bf16* k = reinterpret_cast<const bf16*>(a.k) + (size_t)u * T * kD;
    const bf16* q = reinterpret_cast<const bf16*>(a.q) + (size_t)u * T * kD;
    const bf16* v = reinterpret_cast<const bf16*>(a.v) + (size_t)u * T * kD;
    const bf16* dy = reinterpret_cast<const bf16*>(a.dy) + (size_t)u * T * kD;
    bf16* dk = reinterpret_cast<bf16*>(a.dk) + (size_t)u * T * kD;
    bf16* dq = reinterpret_cast<bf16*>(a.dq) + (size_t)u * T * kD;
    bf16* dv = reinterpret_cast<bf16*>(a.dv) + (size_t)u * T * kD;
    const float* alpha = a.alpha + (size_t)u * T;
    const float* eta = a.eta + (size_t)u * T;
    const float* theta = a.theta + (size_t)u * T;

    // C [128 x N] (+)= A [128 x K] B [N x K]^T at TMEM column `col`; A and B bf16 in global memory,
    // K-major (element (r, k) at p[r * ld + k]) or MN-major (at p[k * ld + r]). Waits for completion.
    auto gemm = [&](uint32_t col, const bf16* pa, size_t lda, bool a_mn, const bf16* pb, size_t ldb, bool b_mn, int N,
                    int K) {
        if (!ok) return;
        tc_fence_before();
        __syncthreads();
        if (a_mn)
            load_mnmajor(sb, pa, lda, 128, 0, K, K);
        else
            load_kmajor(sb, pa, lda, 128, 128, 0, K);
        if (b_mn)
            load_mnmajor(sb + kBOff, pb, ldb, N, 0, K, K);
        else
            load_kmajor(sb + kBOff, pb, ldb, N, N, 0, K);
        operands_ready();
        if (tid == 0) mma_steps(tmem + col, sb, a_mn, sb + kBOff, b_mn, N, K / 16, false);
        if (tid == 0) umma_commit(bar);
        const bool done = mbar_wait(bar, mma_phase);
        mma_phase ^= 1u;
        if (!done) atomicOr(a.status, kStatusTimeoutMma);
        ok = __syncthreads_or(!done) == 0;
        tc_fence_after();
    };
    auto zero = [&](void* p, size_t bytes) {
        uint4* x = reinterpret_cast<uint4*>(p);
        for (size_t i = tid; i < bytes / 16; i += kThreads) x[i] = make_uint4(0, 0, 0, 0);
    };
    // Gate scan of a chunk on warp 0, division-free, two tokens per lane (tokens j >= n are padding:
    // they leave every product unchanged and get c_j = d_j = 0):
    //   P_j = prod_{l>j} (1 - alpha_l), Q_j = prod_{l>j} eta_l,
    //   r_j = P_j + eta_{j+1} r_{j+1} (r_{n-1} = 1; an affine suffix recurrence, scanned by composing
    //   the maps r -> a r + b), c_j = theta_j r_j, d_j = theta_j Q_j,
    //   A = prod_l (1 - alpha_l), E = prod_l eta_l, sigma = eta_0 r_0.
    auto scan = [&](long t0, int n) {
        if (warp == 0) {
            const unsigned FULL = 0xffffffffu;
            const int j0 = 2 * lane, j1 = j0 + 1;
            const float a0 = j0 < n ? alpha[t0 + j0] : 0.f, a1 = j1 < n ? alpha[t0 + j1] : 0.f;
            const float e0 = j0 < n ? eta[t0 + j0] : 1.f, e1 = j1 < n ? eta[t0 + j1] : 1.f;
            const float th0 = j0 < n ? theta[t0 + j0] : 0.f, th1 = j1 < n ? theta[t0 + j1] : 0.f;
            const float om0 = 1.f - a0, om1 = 1.f - a1;
            float pp = om0 * om1, pq = e0 * e1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float x = __shfl_down_sync(FULL, pp, off), y = __shfl_down_sync(FULL, pq, off);
                if (lane + off < 32) {
                    pp *= x;
                    pq *= y;
                }
            }
            float exP = __shfl_down_sync(FULL, pp, 1), exQ = __shfl_down_sync(FULL, pq, 1);
            if (lane == 31) exP = exQ = 1.f;
            const float P1 = exP, P0 = exP * om1, Q1 = exQ, Q0 = exQ * e1;
            const float b0 = j0 < n ? P0 : 0.f, b1 = j1 < n ? P1 : 0.f;
            const float c0 = j1 < n ? e1 : 0.f;  // coefficient of r_{j0 + 1} = r_{j1}
            const float e_next = __shfl_down_sync(FULL, e0, 1);
            const float c1 = j1 + 1 < n ? e_next : 0.f;  // coefficient of r_{j1 + 1}
            float A = c0 * c1, Bv = b0 + c0 * b1;  // this lane's pair as one map of r_{j1 + 1}
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float A2 = __shfl_down_sync(FULL, A, off), B2 = __shfl_down_sync(FULL, Bv, off);
                if (lane + off < 32) {
                    Bv = Bv + A * B2;
                    A = A * A2;
                }
            }
            float r_after = __shfl_down_sync(FULL, Bv, 1);
            if (lane == 31) r_after = 0.f;
            const float r0 = Bv, r1 = b1 + c1 * r_after;
            s_a[j0] = a0; s_a[j1] = a1;
            s_e[j0] = e0; s_e[j1] = e1;
            s_t[j0] = th0; s_t[j1] = th1;
            s_r[j0] = r0; s_r[j1] = r1;
            s_P[j0] = P0; s_P[j1] = P1;
            s_Q[j0] = Q0; s_Q[j1] = Q1;
            s_c[j0] = th0 * r0; s_c[j1] = th1 * r1;
            s_d[j0] = th0 * Q0; s_d[j1] = th1 * Q1;
            if (lane == 0) {
                s_scal[0] = om0 * P0;
                s_scal[1] = e0 * Q0;
                s_scal[2] = e0 * r0;
            }
        }
        __syncthreads();
    };
    // The chunk's token operands: [K; Q], [c K | d K] and (pass 2) dy in rows 64..127 of GQ.
    auto load_chunk = [&](long t0, int n, bool with_dy) {
        for (int i = tid; i < 128 * 8; i += kThreads) {
            const int r = i >> 3, p = i & 7;
            const int t = r & 63;
            const bf16* src = r < 64 ? k : q;
            uint4 x = make_uint4(0, 0, 0, 0);
            if (t < n) x = *reinterpret_cast<const uint4*>(src + (t0 + t) * kD + 8 * p);
            reinterpret_cast<uint4*>(XQ)[i] = x;
        }
        for (int i = tid; i < 64 * 16; i += kThreads) {
            const int r = i >> 4, p = i & 15, which = p >> 3;
            uint4 o = make_uint4(0, 0, 0, 0);
            if (r < n) {
                const float s = which ? s_d[r] : s_c[r];
                const uint4 x = *reinterpret_cast<const uint4*>(k + (t0 + r) * kD + 8 * (p & 7));
                const uint32_t w[4] = {x.x, x.y, x.z, x.w};
                uint32_t y[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = unpack_bf16x2(w[e]);
                    y[e] = pack2(s * f.x, s * f.y);
                }
                o = make_uint4(y[0], y[1], y[2], y[3]);
            }
            reinterpret_cast<uint4*>(CK + (size_t)r * 2 * kD)[p] = o;
            reinterpret_cast<uint4*>(CK + (size_t)(r + 64) * 2 * kD)[p] = o;  // copy in rows 64..127 (below)
        }
        if (with_dy)
            for (int i = tid; i < 64 * 8; i += kThreads) {
                const int r = i >> 3, p = i & 7;
                uint4 x = make_uint4(0, 0, 0, 0);
                if (r < n) x = *reinterpret_cast<const uint4*>(dy + (t0 + r) * kD + 8 * p);
                reinterpret_cast<uint4*>(GQ + (size_t)(64 + r) * kD)[p] = x;
            }
    };
    // bf16 copies of the chunk-start W1, W2. The 128 KB of fp32 come into the (idle) operand region of
    // shared memory with every copy in flight at once, then go out converted.
    auto state_bf16 = [&](const float* X) {
        const uint8_t* src = reinterpret_cast<const uint8_t*>(X);
        for (uint32_t o = 16u * tid; o < 2u * kHD * 4u; o += 16u * kThreads) cp_async16(sb + o, src + o);
        cp_async_wait_all();
        __syncthreads();
        const float4* s4 = reinterpret_cast<const float4*>(sm);
#pragma unroll 4
        for (size_t i = tid; i < kHD / 4; i += kThreads) {
            const float4 w1 = s4[i], w2 = s4[kHD / 4 + i];
            reinterpret_cast<uint2*>(W1b)[i] = make_uint2(pack2(w1.x, w1.y), pack2(w1.z, w1.w));
            reinterpret_cast<uint2*>(W2b)[i] = make_uint2(pack2(w2.x, w2.y), pack2(w2.z, w2.w));
        }
        __syncthreads();
    };
    // Keys' (and in pass 2 queries') forward at the chunk-start weights: silu and its derivatives,
    // G = 2 (Y - v) with its c-, d-scaled copy, B = G W2 and Delta = B * silu'(Z); pass 2 also
    // dzq = (W2^T dy) * silu'(Z_Q).
    auto forward = [&](long t0, int n, bool pass2) {
        gemm(0, XQ, kD, false, W1b, kD, false, kH, kD);  // Z = [K; Q] W1^T
        if (!ok) return;
#pragma unroll 1
        for (int blk = 0; blk < 8; ++blk) {
            const int col = 128 * half + 16 * blk;
            float z[16], o1[16], o2[16], o3[16];
            tmem16(tmem + lane_off + col, z);
            if (row >= 64 && !pass2) continue;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float s = fmaf(0.5f, tanh_approx(0.5f * z[e]), 0.5f);
                const float av = z[e] * s;
                o1[e] = av;
                o2[e] = s + av * (1.f - s);                                  // silu'
                o3[e] = s * (1.f - s) * (2.f + z[e] * (1.f - 2.f * s));      // silu''
            }
            if (row < 64) {
                st16_bf16(PQ + (size_t)(128 + row) * kH + col, o1);
                stcol16(SP, col, row, o2);
                if (pass2) stcol16(SPP, col, row, o3);
            } else {
                st16_bf16(PQ + (size_t)row * kH + col, o1);
                stcol16(SPQ, col, row - 64, o2);
            }
        }
        gemm(256, PQ + (size_t)64 * kH, kH, false, W2b, kH, false, kD, kH);  // [A_q; A] W2^T
        if (!ok) return;
        if (row >= 64) {
            const int t = row - 64;
            const float cr = s_c[t], dr = s_d[t];
#pragma unroll 1
            for (int blk = 0; blk < 2; ++blk) {
                const int col = 32 * half + 16 * blk;
                float y[16], vv[16] = {}, g[16], gc[16], gd[16];
                tmem16(tmem + lane_off + 256 + col, y);
                if (t < n) ld16_bf16(v + (t0 + t) * kD + col, vv);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    g[e] = t < n ? 2.f * (y[e] - vv[e]) : 0.f;
                    gc[e] = cr * g[e];
                    gd[e] = dr * g[e];
                }
                stcol16(GF, col, t, g);
                st16_bf16(GQ + (size_t)t * kD + col, g);
                st16_bf16(CG + (size_t)t * 2 * kD + col, gc);
                st16_bf16(CG + (size_t)t * 2 * kD + kD + col, gd);
                st16_bf16(CG + (size_t)(64 + t) * 2 * kD + col, gc);  // copy in rows 64..127 (below)
                st16_bf16(CG + (size_t)(64 + t) * 2 * kD + kD + col, gd);
            }
        }
        gemm(0, GQ, kD, false, W2b, kH, true, kH, kD);  // [G; dy] W2
        if (!ok) return;
#pragma unroll 1
        for (int blk = 0; blk < 8; ++blk) {
            const int col = 128 * half + 16 * blk;
            float b[16], s[16], o[16];
            tmem16(tmem + lane_off + col, b);
            if (row < 64) {
                ldcol16(SP, col, row, s);
#pragma unroll
                for (int e = 0; e < 16; ++e) o[e] = b[e] * s[e];
                st16_bf16(DL + (size_t)row * kH + col, o);
                if (pass2) stcol16(BM, col, row, b);
            } else if (pass2) {
                ldcol16(SPQ, col, row - 64, s);
#pragma unroll
                for (int e = 0; e < 16; ++e) o[e] = b[e] * s[e];
                st16_bf16(DZ + (size_t)row * kH + col, o);
            }
        }
    };

    // ---- set-up: zero the operand buffers (padding rows stay zero), chunk 0's state
    zero(XQ, (size_t)128 * kD * 2);
    zero(CK, (size_t)128 * 2 * kD * 2);
    zero(PQ, (size_t)256 * kH * 2);
    zero(GQ, (size_t)256 * kD * 2);
    zero(CG, (size_t)128 * 2 * kD * 2);
    zero(DZ, (size_t)128 * kH * 2);
    zero(DL, (size_t)128 * kH * 2);
    if (!a.ckpt_ready)
        for (size_t i = tid; i < 4 * kHD; i += kThreads) {
            const float* src = i < kHD ? a.W1 : (i < 2 * kHD ? a.W2 : (i < 3 * kHD ? a.S1 : a.S2));
            ckpt[i] = src[u * kHD + (i % kHD)];
        }
    __syncthreads();

    // ---- pass 1: the forward, keeping each chunk-start state (unless the chunk kernel already
    //      wrote them into the workspace)
    for (long c = 0; c + 1 < nch && ok && !a.ckpt_ready; ++c) {
        const long t0 = c * chunk;
        const int n = (int)min((long)chunk, T - t0);
        const float* X = ckpt + (size_t)c * 4 * kHD;
        float* Xn = ckpt + (size_t)(c + 1) * 4 * kHD;
        if (!DBG(n >= 1 && n <= kN)) break;  // the same outcome in every thread
        scan(t0, n);
        load_chunk(t0, n, false);
        state_bf16(X);
        forward(t0, n, false);
        // [dW1_c | dW1_d] = Delta^T [c K | d K] (cols 128 mt), [dW2_c^T | dW2_d^T] = A^T [c G | d G]
        // (cols 256 + 128 mt), per 128 hidden rows mt
        for (int mt = 0; mt < 2; ++mt) {
            gemm(128 * mt, DL + 128 * mt, kH, true, CK, 2 * kD, true, 2 * kD, kN);
            gemm(256 + 128 * mt, PQ + (size_t)128 * kH + 128 * mt, kH, true, CG, 2 * kD, true, 2 * kD, kN);
        }
        if (!ok) break;
        const float An = s_scal[0], En = s_scal[1], sig = s_scal[2];
        // The accumulators go through shared memory (rows of 65 floats) so that the state update
        // reads and writes W, S with consecutive threads on consecutive elements. W1 and S1 first
        // (TMEM columns 128 mt: c part, + 64: d part), then W2 and S2 (columns 256 + 128 mt).
        float* st_c = reinterpret_cast<float*>(sm);
        float* st_d = st_c + 256 * 65;
        for (int part = 0; part < 2; ++part) {
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            for (int mt = 0; mt < 2; ++mt) {
                const int j = 128 * mt + row;
#pragma unroll 1
                for (int blk = 0; blk < 2; ++blk) {
                    const int col = 32 * half + 16 * blk;
                    float ac[16], ad[16];
                    tmem16(tmem + lane_off + 256 * part + 128 * mt + col, ac);
                    tmem16(tmem + lane_off + 256 * part + 128 * mt + kD + col, ad);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        st_c[j * 65 + col + e] = ac[e];
                        st_d[j * 65 + col + e] = ad[e];
                    }
                }
            }
            __syncthreads();
            // four consecutive elements per thread and step (float4 global accesses)
            const size_t o = part == 0 ? 0 : kHD;
#pragma unroll 4
            for (size_t i = 4 * tid; i < kHD; i += 4 * kThreads) {
                const float4 w = *reinterpret_cast<const float4*>(X + o + i);
                const float4 sv = *reinterpret_cast<const float4*>(X + 2 * kHD + o + i);
                float ac[4], ad[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    // W1, S1 [h][d]: element (j, m) = (i / d, i % d); W2, S2 [d][h]: (r, j) = (i / h, i % h)
                    const size_t at = part == 0 ? (i / kD) * 65 + (i % kD) + e : ((i % kH) + e) * 65 + i / kH;
                    ac[e] = st_c[at];
                    ad[e] = st_d[at];
                }
                *reinterpret_cast<float4*>(Xn + o + i) =
                    make_float4(fmaf(An, w.x, sig * sv.x) - ac[0], fmaf(An, w.y, sig * sv.y) - ac[1],
                                fmaf(An, w.z, sig * sv.z) - ac[2], fmaf(An, w.w, sig * sv.w) - ac[3]);
                *reinterpret_cast<float4*>(Xn + 2 * kHD + o + i) =
                    make_float4(En * sv.x - ad[0], En * sv.y - ad[1], En * sv.z - ad[2], En * sv.w - ad[3]);
            }
        }
        __syncthreads();
    }

    // ---- pass 2: backwards
    // The adjoint dW1', dW2', dS1', dS2' at the chunk's end; the update below turns it into the
    // chunk-start adjoint in place (each element is read, then written, by the same thread).
    float* dcur = adj;
    for (size_t i = tid; i < 4 * kHD; i += kThreads) {
        const float* src = i < kHD ? a.dW1 : (i < 2 * kHD ? a.dW2 : (i < 3 * kHD ? a.dS1 : a.dS2));
        dcur[i] = src ? src[u * kHD + (i % kHD)] : 0.f;
    }
    __syncthreads();
    for (size_t i = tid; i < kHD; i += kThreads) {
        const size_t j = i / kD, m = i % kD;  // dW1', dS1' row j interleaved; dW2', dS2' stacked
        dW1b[j * 2 * kD + m] = __float2bfloat16_rn(dcur[i]);
        dW1b[j * 2 * kD + kD + m] = __float2bfloat16_rn(dcur[2 * kHD + i]);
        dW2b[i] = __float2bfloat16_rn(dcur[kHD + i]);
        dW2b[kHD + i] = __float2bfloat16_rn(dcur[3 * kHD + i]);
    }
    __syncthreads();
    for (long c = nch - 1; c >= 0 && ok; --c) {
        const long t0 = c * chunk;
        const int n = (int)min((long)chunk, T - t0);
        const float* X = ckpt + (size_t)c * 4 * kHD;
        if (!DBG(n >= 1 && n <= kN)) break;
        scan(t0, n);
        load_chunk(t0, n, true);
        state_bf16(X);
        forward(t0, n, true);

        // dG0 = -(c A dW2'^T + d A dS2'^T); dc, dd from -g . (dW2' a), -g . (dS2' a)
        // (one N = 128 GEMM: rows 0..63 of [dW2'; dS2'] land in columns 256.., rows 64..127 in 256 + d..)
        gemm(256, PQ + (size_t)128 * kH, kH, false, dW2b, kH, false, 2 * kD, kH);
        if (!ok) break;
        {
            float pc = 0.f, pd = 0.f;
            if (row < 64) {
                const int t = row;
#pragma unroll 1
                for (int blk = 0; blk < 2; ++blk) {
                    const int col = 32 * half + 16 * blk;
                    float x2[16], y2[16], g[16], o[16];
                    tmem16(tmem + lane_off + 256 + col, x2);
                    tmem16(tmem + lane_off + 256 + kD + col, y2);
                    ldcol16(GF, col, t, g);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        o[e] = -(s_c[t] * x2[e] + s_d[t] * y2[e]);
                        pc -= g[e] * x2[e];
                        pd -= g[e] * y2[e];
                    }
                    stcol16(DG0, col, t, o);
                }
            }
            s_part[half * 128 + row] = pc;
            s_part[256 + half * 128 + row] = pd;
            __syncthreads();
            if (tid < 64) {
                s_dc[tid] = s_part[tid] + s_part[128 + tid];
                s_dd[tid] = s_part[256 + tid] + s_part[384 + tid];
            }
        }
        // dA0 = -[c G | d G] [dW2'; dS2'];  ddelta = -[c K | d K] [dW1' | dS1']^T -> db, dz0
        // Rows 64..127 of [c G | d G] and [c K | d K] repeat rows 0..63, so TMEM lanes 64..127 hold a
        // second copy of the products and all eight warps share the epilogue: lanes 0..63 take the
        // first four 16-column blocks of their half, lanes 64..127 the last four.
        gemm(0, CG, 2 * kD, false, dW2b, kH, true, kH, 2 * kD);
        gemm(256, CK, 2 * kD, false, dW1b, 2 * kD, false, kH, 2 * kD);
        if (!ok) break;
        {
            const int t = row & 63, sub = row >> 6;
#pragma unroll 1
            for (int blk = 4 * sub; blk < 4 * sub + 4; ++blk) {
                const int col = 128 * half + 16 * blk;
                float x[16], y[16], s[16], b[16], s2[16], o[16];
                tmem16(tmem + lane_off + col, x);
#pragma unroll
                for (int e = 0; e < 16; ++e) o[e] = -x[e];
                stcol16(DA0, col, t, o);
                tmem16(tmem + lane_off + 256 + col, y);
                ldcol16(SP, col, t, s);
                ldcol16(BM, col, t, b);
                ldcol16(SPP, col, t, s2);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float ddel = -y[e];
                    o[e] = ddel * s[e];     // db
                    x[e] = ddel * b[e] * s2[e];  // dz0
                }
                st16_bf16(PQ + (size_t)t * kH + col, o);
                stcol16(DZ0, col, t, x);
            }
        }
        // dG = dG0 + db W2^T; dyhat = 2 dG, dv = -2 dG
        gemm(0, PQ, kH, false, W2b, kH, false, kD, kH);
        if (!ok) break;
        if (row < 64) {
            const int t = row;
#pragma unroll 1
            for (int blk = 0; blk < 2; ++blk) {
                const int col = 32 * half + 16 * blk;
                float x[16], g0[16], o[16], ov[16];
                tmem16(tmem + lane_off + col, x);
                ldcol16(DG0, col, t, g0);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float g = g0[e] + x[e];
                    o[e] = 2.f * g;
                    ov[e] = -2.f * g;
                }
                st16_bf16(GQ + (size_t)(128 + t) * kD + col, o);
                st16_bf16(GQ + (size_t)(192 + t) * kD + col, o);  // copy in rows 192..255 (below)
                if (t < n && DBG(t0 + t < T)) st16_bf16(dv + (t0 + t) * kD + col, ov);
            }
        }
        // dA = dA0 + dyhat W2;  dz = dz0 + dA * silu'(Z)
        // (rows 192..255 of GQ repeat dyhat: lanes 64..127 hold a copy, shared out as above)
        gemm(0, GQ + (size_t)128 * kD, kD, false, W2b, kH, true, kH, kD);
        if (!ok) break;
        {
            const int t = row & 63, sub = row >> 6;
#pragma unroll 1
            for (int blk = 4 * sub; blk < 4 * sub + 4; ++blk) {
                const int col = 128 * half + 16 * blk;
                float x[16], a0[16], s[16], z0[16], o[16];
                tmem16(tmem + lane_off + col, x);
                ldcol16(DA0, col, t, a0);
                ldcol16(SP, col, t, s);
                ldcol16(DZ0, col, t, z0);
#pragma unroll
                for (int e = 0; e < 16; ++e) o[e] = z0[e] + (a0[e] + x[e]) * s[e];
                st16_bf16(DZ + (size_t)t * kH + col, o);
            }
        }
        // dk = -(c Delta dW1' + d Delta dS1') + dz W1, dq = dzq W1; dc, dd from -k . (Delta dW1'), ...
        // (one N = 128 GEMM for Delta [dW1' | dS1']: columns 0.. and d..)
        gemm(0, DL, kH, false, dW1b, 2 * kD, true, 2 * kD, kH);
        gemm(2 * kD, DZ, kH, false, W1b, kD, true, kD, kH);
        if (!ok) break;
        {
            float pc = 0.f, pd = 0.f;
            const int t = row & 63;
#pragma unroll 1
            for (int blk = 0; blk < 2; ++blk) {
                const int col = 32 * half + 16 * blk;
                float x0[16], x1[16], x2[16], km[16], o[16];
                tmem16(tmem + lane_off + 2 * kD + col, x2);
                if (row < 64) {
                    tmem16(tmem + lane_off + col, x0);
                    tmem16(tmem + lane_off + kD + col, x1);
                    ld16_bf16(XQ + (size_t)t * kD + col, km);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        o[e] = -(s_c[t] * x0[e] + s_d[t] * x1[e]) + x2[e];
                        pc -= km[e] * x0[e];
                        pd -= km[e] * x1[e];
                    }
                    if (t < n && DBG(t0 + t < T)) st16_bf16(dk + (t0 + t) * kD + col, o);
                } else if (t < n && DBG(t0 + t < T)) {
                    st16_bf16(dq + (t0 + t) * kD + col, x2);
                }
            }
            s_part[half * 128 + row] = pc;
            s_part[256 + half * 128 + row] = pd;
            __syncthreads();
            if (tid < 64) {
                s_dc[tid] += s_part[tid] + s_part[128 + tid];
                s_dd[tid] += s_part[256 + tid] + s_part[384 + tid];
            }
        }
        // chunk-start adjoints: dW1 = A dW1' + [dz; dzq]^T [K; Q], dW2^T = A dW2'^T + [db; A_q; A]^T [G; dy; dyhat],
        // dS = sigma dW' + E dS'; and the chunk scalars' adjoints <dW', W>, <dW', S>, <dS', S>
        // The adjoint update below streams this chunk's checkpoint and the adjoint (256 KB each): they
        // start moving into L2 now, while the four GEMMs run (16 KB pieces).
        if (tid == 0)
            for (int piece = 0; piece < 16; ++piece) {
                prefetch_l2_bulk(X + (size_t)piece * kHD / 4, (uint32_t)(kHD / 4 * sizeof(float)));
                prefetch_l2_bulk(dcur + (size_t)piece * kHD / 4, (uint32_t)(kHD / 4 * sizeof(float)));
            }
        for (int mt = 0; mt < 2; ++mt) {
            gemm(kD * mt, DZ + 128 * mt, kH, true, XQ, kD, true, kD, 128);
            gemm(2 * kD + kD * mt, PQ + 128 * mt, kH, true, GQ, kD, true, kD, 192);
        }
        if (!ok) break;
        {
            const float An = s_scal[0], En = s_scal[1], sig = s_scal[2];
            // The accumulators (dW1 tiles at TMEM columns 64 mt, dW2^T tiles at 128 + 64 mt) go through
            // shared memory (rows of 65 floats); the adjoint update then runs with consecutive threads
            // on consecutive elements.
            float* st1 = reinterpret_cast<float*>(sm);
            float* st2 = st1 + 256 * 65;
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            for (int mt = 0; mt < 2; ++mt) {
                const int j = 128 * mt + row;
#pragma unroll 1
                for (int blk = 0; blk < 2; ++blk) {
                    const int col = 32 * half + 16 * blk;
                    float x1[16], x2[16];
                    tmem16(tmem + lane_off + kD * mt + col, x1);
                    tmem16(tmem + lane_off + 2 * kD + kD * mt + col, x2);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        st1[j * 65 + col + e] = x1[e];
                        st2[j * 65 + col + e] = x2[e];
                    }
                }
            }
            __syncthreads();
            float pa = 0.f, ps = 0.f, pe = 0.f;
            // four consecutive elements per thread and step (float4 global accesses)
            for (int part = 0; part < 2; ++part) {
                const size_t o = part == 0 ? 0 : kHD;
                const float* st = part == 0 ? st1 : st2;
#pragma unroll 8
                for (size_t i = 4 * tid; i < kHD; i += 4 * kThreads) {
                    const float4 dw = *reinterpret_cast<const float4*>(dcur + o + i);
                    const float4 ds = *reinterpret_cast<const float4*>(dcur + 2 * kHD + o + i);
                    const float4 w = *reinterpret_cast<const float4*>(X + o + i);
                    const float4 sv = *reinterpret_cast<const float4*>(X + 2 * kHD + o + i);
                    const float dwv[4] = {dw.x, dw.y, dw.z, dw.w}, dsv[4] = {ds.x, ds.y, ds.z, ds.w};
                    const float wv[4] = {w.x, w.y, w.z, w.w}, svv[4] = {sv.x, sv.y, sv.z, sv.w};
                    float nw[4], ns[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const size_t at = part == 0 ? (i / kD) * 65 + (i % kD) + e : ((i % kH) + e) * 65 + i / kH;
                        nw[e] = fmaf(An, dwv[e], st[at]);
                        ns[e] = fmaf(sig, dwv[e], En * dsv[e]);
                        pa += dwv[e] * wv[e];
                        ps += dwv[e] * svv[e];
                        pe += dsv[e] * svv[e];
                    }
                    *reinterpret_cast<float4*>(dcur + o + i) = make_float4(nw[0], nw[1], nw[2], nw[3]);
                    *reinterpret_cast<float4*>(dcur + 2 * kHD + o + i) = make_float4(ns[0], ns[1], ns[2], ns[3]);
                    const uint2 bw = make_uint2(pack2(nw[0], nw[1]), pack2(nw[2], nw[3]));
                    const uint2 bs = make_uint2(pack2(ns[0], ns[1]), pack2(ns[2], ns[3]));
                    if (part == 0) {  // [h][dW1' | dS1'], row j = i / d
                        *reinterpret_cast<uint2*>(dW1b + (i / kD) * 2 * kD + (i % kD)) = bw;
                        *reinterpret_cast<uint2*>(dW1b + (i / kD) * 2 * kD + kD + (i % kD)) = bs;
                    } else {          // [dW2'; dS2']
                        *reinterpret_cast<uint2*>(dW2b + i) = bw;
                        *reinterpret_cast<uint2*>(dW2b + kHD + i) = bs;
                    }
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                pa += __shfl_xor_sync(0xffffffffu, pa, off);
                ps += __shfl_xor_sync(0xffffffffu, ps, off);
                pe += __shfl_xor_sync(0xffffffffu, pe, off);
            }
            if (lane == 0) {
                s_red[4 * warp] = pa;
                s_red[4 * warp + 1] = ps;
                s_red[4 * warp + 2] = pe;
            }
            __syncthreads();
        }
        if (tid == 0) {
            // The next chunk back (a full one): the weights half of its checkpoint and its token rows,
            // which its set-up reads first. Issued this late they measured faster than at the
            // chunk's start, where the prefetched lines compete with the chunk's own working set.
            if (c > 0) {
                const float* xn = ckpt + (size_t)(c - 1) * 4 * kHD;
                for (int piece = 0; piece < 8; ++piece)
                    prefetch_l2_bulk(xn + (size_t)piece * kHD / 4, (uint32_t)(kHD / 4 * sizeof(float)));
                const long tp = (c - 1) * chunk;
                const uint32_t rows = (uint32_t)chunk * kD * 2;
                prefetch_l2_bulk(k + tp * kD, rows);
                prefetch_l2_bulk(q + tp * kD, rows);
                prefetch_l2_bulk(v + tp * kD, rows);
                prefetch_l2_bulk(dy + tp * kD, rows);
            }
        }
        // The gates' adjoints through the scan, on warp 0 (two tokens per lane). With dr_{-1} = dsig:
        //   dr_j = theta_j dc_j + eta_j dr_{j-1},
        //   F_0 = dA, F_{j+1} = (1 - alpha_j) F_j + dr_j;  H_0 = dE, H_{j+1} = eta_j H_j + theta_j dd_j,
        //   dtheta_j = dc_j r_j + dd_j Q_j, dalpha_j = -P_j F_j, deta_j = Q_j H_j + dr_{j-1} r_j.
        // Each recurrence is a prefix scan of affine maps x -> a x + b over the lanes.
        if (warp == 0) {
            const unsigned FULL = 0xffffffffu;
            float dA = 0.f, dsig = 0.f, dE = 0.f;
            for (int w = 0; w < kThreads / 32; ++w) {
                dA += s_red[4 * w];
                dsig += s_red[4 * w + 1];
                dE += s_red[4 * w + 2];
            }
            const int j0 = 2 * lane, j1 = j0 + 1;
            const bool in0 = j0 < n, in1 = j1 < n;
            // padding tokens take the identity map
            const float e0 = in0 ? s_e[j0] : 1.f, e1 = in1 ? s_e[j1] : 1.f;
            const float om0 = in0 ? 1.f - s_a[j0] : 1.f, om1 = in1 ? 1.f - s_a[j1] : 1.f;
            const float g0 = in0 ? s_t[j0] * s_dc[j0] : 0.f, g1 = in1 ? s_t[j1] * s_dc[j1] : 0.f;
            const float h0 = in0 ? s_t[j0] * s_dd[j0] : 0.f, h1 = in1 ? s_t[j1] * s_dd[j1] : 0.f;
            // inclusive prefix over lanes of the pair maps (later map after earlier: a = a2 a1, b = a2 b1 + b2),
            // then the exclusive value at the lane's first token
            auto prefix = [&](float a, float b, float x0) {
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float ap = __shfl_up_sync(FULL, a, off), bp = __shfl_up_sync(FULL, b, off);
                    if (lane >= off) {
                        b = a * bp + b;
                        a = a * ap;
                    }
                }
                float ae = __shfl_up_sync(FULL, a, 1), be = __shfl_up_sync(FULL, b, 1);
                if (lane == 0) {
                    ae = 1.f;
                    be = 0.f;
                }
                return ae * x0 + be;
            };
            const float dr_in = prefix(e1 * e0, e1 * g0 + g1, dsig);  // dr_{j0 - 1}
            const float dr0 = e0 * dr_in + g0, dr1 = e1 * dr0 + g1;
            const float F0 = prefix(om1 * om0, om1 * dr0 + dr1, dA), F1 = om0 * F0 + dr0;
            const float H0 = prefix(e1 * e0, e1 * h0 + h1, dE), H1 = e0 * H0 + h0;
            const long g = u * T + t0;
            if (in0) {
                a.dtheta[g + j0] = s_dc[j0] * s_r[j0] + s_dd[j0] * s_Q[j0];
                a.dalpha[g + j0] = -s_P[j0] * F0;
                a.deta[g + j0] = s_Q[j0] * H0 + dr_in * s_r[j0];
            }
            if (in1) {
                a.dtheta[g + j1] = s_dc[j1] * s_r[j1] + s_dd[j1] * s_Q[j1];
                a.dalpha[g + j1] = -s_P[j1] * F1;
                a.deta[g + j1] = s_Q[j1] * H1 + dr0 * s_r[j1];
            }
        }
        __syncthreads();
    }
    if (ok)
        for (size_t i = tid; i < 4 * kHD; i += kThreads) {
            float* dst = i < kHD ? a.dW1_0 : (i < 2 * kHD ? a.dW2_0 : (i < 3 * kHD ? a.dS1_0 : a.dS2_0));
            dst[u * kHD + (i % kHD)] = dcur[i];
        }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

#undef DBG

bool mlp_backward_tc_supported(int d, int h, int chunk) {
    return d == mbt::kD && h == mbt::kH && chunk >= 1 && chunk <= mbt::kN;
}

size_t mlp_backward_tc_ckpt_offset() { return mbt::layout(1).ckpt; }

size_t mlp_backward_tc_ws_bytes(long T, int chunk) {
    if (chunk < 1) return 0;
    return mbt::layout((T + chunk - 1) / chunk).total;
}

cudaError_t launch_mlp_backward_tc(const MlpBackwardArgs& a, cudaStream_t st) {
    if (!a.bf16 || !mlp_backward_tc_supported(a.d, a.h, a.chunk)) return cudaErrorInvalidValue;
    if (a.ws_per_unit * sizeof(float) < mlp_backward_tc_ws_bytes(a.T, a.chunk)) return cudaErrorInvalidValue;
    static std::atomic<unsigned> attr_set{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 32) return cudaErrorInvalidDevice;
    if (!(attr_set.load() & (1u << dev))) {
        e = cudaFuncSetAttribute(mlp_backward_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)mbt::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(1u << dev);
    }
    mlp_backward_tc_kernel<<<(unsigned)a.units, mbt::kThreads, mbt::kSmemBytes, st>>>(a);
    return cudaGetLastError();
}

}  // namespace titans
