// Tensor-core chunk forward of the deep memory M(x) = W_L silu(W_{L-1} ... silu(W_1 x)), L >= 3
// layers, width d in {64, 128}, hidden width h = 4d, chunk n <= 128, bf16 operands with fp32
// accumulation, fp32 state.
//
// Method ("Titans: Learning to Memorize at Test Time", walk-through sec. 3.1 "Memory Architecture",
// sec. 5.5 "The Effect of Deep Memory"; sec. 3.2 for the chunk-wise form): every token of a chunk
// takes its gradient of ||M(k) - v||^2 at the chunk-start weights of every layer, so each layer's
// momentum and forgetting recurrence folds into
//   W_l <- A W_l + sigma S_l - sum_j c_j g_{l,j},   S_l <- E S_l - sum_j d_j g_{l,j},
// with c_j, d_j, A, E, sigma from the division-free suffix scan of the gates, and the sums of
// per-token outer products g_{l,j} = delta_{l,j} a_{l-1,j}^T are weighted GEMMs.
//
// A unit's state does not fit one SM (768 KB at d = 64 with four layers), so, like the wide
// 2-layer kernel, one persistent CTA per SM walks every unit's chunks in grid-wide phases of
// 128-row tcgen05 tiles, with the state and intermediates in L2 between phases. Per chunk:
//   F_1 ... F_{L-1}  Z_l^T = W_l A_{l-1}^T (A_0 = [K; Q]), keys and queries as separate 128-token
//                    tiles -> A_l^T = silu(Z_l)^T (bf16) and, for the keys, silu'(Z_l)^T (fp32);
//                    F_1 also runs the gate scan, one tile per unit.
//   OUT              Y = A_{L-1} W_L^T -> keys: G = 2 (Y - v) and -c G, -d G; queries: y (or the
//                    gated output attn * sigmoid(y)).
//   B_L ... B_2      Delta_{L-1}^T = (W_L^T G^T) * silu'(Z_{L-1})^T, then
//                    Delta_{l-1}^T = (W_l^T Delta_l^T) * silu'(Z_{l-1})^T; each written unscaled
//                    (the next step's operand) and as Delta^T diag(-c), Delta^T diag(-d).
//   WGT              every layer's dW_{l,c} and dW_{l,d} (two TMEM accumulators per tile) and the
//                    fp32 update of W_l, S_l, with the bf16 copy of W_l the next chunk reads.
//                    The last layer's tiles are computed transposed (dW_L^T, 128 hidden rows).
// The phases are separated by the bounded grid barrier; the kernel is launched cooperatively.
#include <cuda_bf16.h>

#include <atomic>
#include <cstdint>

#include "kernels.h"
#include "phased_common.cuh"
#include "ptx.cuh"

namespace titans {

namespace dp {
using phc::kThreads;
constexpr int kNmax = 128;
constexpr int kKc = 256;  // K elements per operand round of the forward and back-propagation tiles
constexpr uint32_t kSmemOperands = 224 * 1024;
constexpr uint32_t kStageW = 96 * 1024, kStageS = 160 * 1024;  // fp32 state tiles of the weight phase
constexpr uint32_t kSpS = 128 * 1024;                         // silu' rows of a back-propagation tile
constexpr uint32_t kScS = 192 * 1024;                         // c, d of the chunk (back-propagation tiles)
constexpr uint32_t kInS = 192 * 1024;                         // v or attn rows of an output tile
constexpr uint32_t BAR = kSmemOperands;
constexpr uint32_t TPTR = BAR + 8;
constexpr uint32_t OKF = TPTR + 4;
constexpr uint32_t END = OKF + 4;
constexpr size_t kSmemBytes = END + 1024;
constexpr uint32_t kTmemCols = 256;  // two accumulators of up to 128 columns
}  // namespace dp

static_assert(dp::kSmemBytes <= 232448, "shared memory budget");

struct DeepTcArgs {
    const __nv_bfloat16 *k, *q, *v;
    const float *alpha, *eta, *theta;
    float *W, *S;  // [units][P] fp32, layers packed W_1 [h][d], W_2 .. W_{L-1} [h][h], W_L [d][h]
    __nv_bfloat16* y;
    const __nv_bfloat16* attn;
    uint8_t* ws;
    size_t ws_stride;  // bytes per unit
    long T, gate_ld, P;
    int chunk, units, D, H, L;
    int chunk_gates;
    // byte offsets of the pieces of a unit's workspace
    size_t o_wb, o_act, o_sp, o_dlt, o_dlc, o_dld, o_gg, o_gc, o_gd, o_sc;
    unsigned* status;
    unsigned* sync;  // [0] barrier arrivals, [1] abort flag; zero at launch
};

namespace {

using phc::desc_k;
using phc::desc_mn;
using phc::load_kmajor;
using phc::load_mnmajor;
using phc::load_tile;
using phc::mma_steps;
using phc::operands_ready;
using phc::pack2;
using phc::srow_off;
using phc::stage_rows_in;
using phc::stage_rows_out;
using phc::tanh_approx;

size_t align1k(size_t x) { return (x + 1023) & ~size_t(1023); }

// Workspace layout of one unit; returns its size in bytes.
size_t deep_layout(int D, int H, int L, DeepTcArgs& a) {
    const size_t P = (size_t)2 * D * H + (size_t)(L - 2) * H * H;
    size_t o = 0;
    a.o_wb = o;   // bf16 copy of every layer
    o = align1k(o + P * 2);
    a.o_act = o;  // per hidden layer: silu(Z_l)^T bf16 [h][keys 128 | queries 128]
    o = align1k(o + (size_t)(L - 1) * H * 256 * 2);
    a.o_sp = o;   // per hidden layer: silu'(Z_l,K)^T fp32 [h][128]
    o = align1k(o + (size_t)(L - 1) * H * 128 * 4);
    a.o_dlt = o;  // per hidden layer: Delta_l^T, -c and -d scaled copies, bf16 [h][128] each
    o = align1k(o + (size_t)(L - 1) * H * 128 * 2);
    a.o_dlc = o;
    o = align1k(o + (size_t)(L - 1) * H * 128 * 2);
    a.o_dld = o;
    o = align1k(o + (size_t)(L - 1) * H * 128 * 2);
    a.o_gg = o;   // G, -c G, -d G bf16 [128 tok][d]
    o = align1k(o + (size_t)128 * D * 2);
    a.o_gc = o;
    o = align1k(o + (size_t)128 * D * 2);
    a.o_gd = o;
    o = align1k(o + (size_t)128 * D * 2);
    a.o_sc = o;   // fp32 c[128], d[128], A, E, sigma
    o += 2048;
    return o;
}

__device__ __forceinline__ long woff(const DeepTcArgs& a, int l) {
    return l == 1 ? 0 : (long)a.D * a.H + (long)(l - 2) * a.H * a.H;
}

}  // namespace

__global__ void __launch_bounds__(dp::kThreads, 1) chunk_fwd_tc_deep(const __grid_constant__ DeepTcArgs a) {
    using namespace dp;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + BAR);
    volatile uint32_t* s_ok = reinterpret_cast<volatile uint32_t*>(sm + OKF);
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
    unsigned epoch = 0;
    uint32_t mma_phase = 0;
    bool ok = true;
#define DBG(cond) TITANS_DBG(cond, a.status, reinterpret_cast<volatile int*>(&a.sync[1]))

    auto mma_done = [&]() -> bool {
        if (tid == 0) umma_commit(bar);
        const bool done = mbar_wait(bar, mma_phase);
        mma_phase ^= 1u;
        if (!done) {
            atomicOr(a.status, kStatusTimeoutMma);
            atomicExch(&a.sync[1], 1u);
        }
        const bool all = __syncthreads_or(!done) == 0;
        tc_fence_after();
        return all;
    };
    auto sync = [&]() { return phc::grid_sync(a.sync, a.status, epoch, s_ok); };

    const int units = a.units, D = a.D, H = a.H, L = a.L, HT = H / 128;
    const long T = a.T;
    const int nchunks = (int)((T + a.chunk - 1) / a.chunk);
    auto unit_ws = [&](int u) { return a.ws + (size_t)u * a.ws_stride; };
    auto wb = [&](uint8_t* w, int l) { return reinterpret_cast<__nv_bfloat16*>(w + a.o_wb) + woff(a, l); };
    auto act = [&](uint8_t* w, int l) { return reinterpret_cast<__nv_bfloat16*>(w + a.o_act) + (size_t)(l - 1) * H * 256; };
    auto spp = [&](uint8_t* w, int l) { return reinterpret_cast<float*>(w + a.o_sp) + (size_t)(l - 1) * H * 128; };
    auto dlt = [&](uint8_t* w, size_t o, int l) { return reinterpret_cast<__nv_bfloat16*>(w + o) + (size_t)(l - 1) * H * 128; };
    if (!DBG(D % 64 == 0 && D <= 128 && H % 128 == 0 && H <= 512 && L >= 3 && a.chunk >= 1 && a.chunk <= kNmax))
        ok = false;

    // ---- prologue: bf16 copies of every unit's weights
    for (long i = (long)blockIdx.x * kThreads + tid; i < (long)units * a.P / 4; i += (long)gridDim.x * kThreads) {
        const long e = 4 * i;
        const int u = (int)(e / a.P);
        const long r = e % a.P;
        const float4 x = __ldcg(reinterpret_cast<const float4*>(a.W + e));
        uint2* d = reinterpret_cast<uint2*>(unit_ws(u) + a.o_wb + 2 * r);
        __stcg(d, make_uint2(pack2(x.x, x.y), pack2(x.z, x.w)));
    }
    ok = sync() && ok;

    // Epilogue of a forward tile: TMEM [128 rows of layer l][128 tokens of part p] -> silu (and silu').
    auto forward_epilogue = [&](uint8_t* w, int l, int mt, int p) {
        constexpr uint32_t kAt = 0, kSp = 32 * 1024;
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
            uint32_t r[16];
            tmem_ld16(tmem + lane_off + 64 * half + 16 * blk, r);
            tmem_wait_ld();
            uint32_t pk[8];
            float spv[16];
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                // sigma(z) = (1 + tanh(z / 2)) / 2, silu(z) = z sigma(z), silu'(z) = sigma + silu (1 - sigma)
                const float z0 = __uint_as_float(r[i]), z1 = __uint_as_float(r[i + 1]);
                const float s0 = fmaf(0.5f, tanh_approx(0.5f * z0), 0.5f);
                const float s1 = fmaf(0.5f, tanh_approx(0.5f * z1), 0.5f);
                const float a0 = z0 * s0, a1 = z1 * s1;
                pk[i / 2] = pack2(a0, a1);
                spv[i] = s0 + a0 * (1.f - s0);
                spv[i + 1] = s1 + a1 * (1.f - s1);
            }
            st_shared_v4(sb + kAt + srow_off(row, 8 * half + 2 * blk, 256), pk[0], pk[1], pk[2], pk[3]);
            st_shared_v4(sb + kAt + srow_off(row, 8 * half + 2 * blk + 1, 256), pk[4], pk[5], pk[6], pk[7]);
            if (p == 0) {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    st_shared_v4(sb + kSp + srow_off(row, 16 * half + 4 * blk + q4, 512),
                                 __float_as_uint(spv[4 * q4]), __float_as_uint(spv[4 * q4 + 1]),
                                 __float_as_uint(spv[4 * q4 + 2]), __float_as_uint(spv[4 * q4 + 3]));
            }
        }
        __syncthreads();
        stage_rows_out(sm + kAt, act(w, l) + (size_t)mt * 128 * 256 + p * 128, 256 * 2, 128, 256);
        if (p == 0) stage_rows_out(sm + kSp, spp(w, l) + (size_t)mt * 128 * 128, 128 * 4, 128, 512);
    };

    // Epilogue of a back-propagation tile: TMEM [128 rows of layer l][128 tokens] * silu'(Z_l)^T ->
    // Delta_l^T (kept when a further layer reads it) and its -c, -d scaled copies.
    auto backprop_epilogue = [&](uint8_t* w, int l, int mt) {
        constexpr uint32_t kDt = 0, kDc = 32 * 1024, kDd = 64 * 1024;
        const float* s_sc = reinterpret_cast<const float*>(sm + kScS);
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
            const int col = 64 * half + 16 * blk;  // first token of the block
            uint32_t r[16];
            tmem_ld16(tmem + lane_off + col, r);
            tmem_wait_ld();
            uint32_t pt[8], pc[8], pd[8];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const uint4 sp = ld_shared_v4(sb + kSpS + srow_off(row, col / 4 + q4, 512));
                const float spf[4] = {__uint_as_float(sp.x), __uint_as_float(sp.y), __uint_as_float(sp.z),
                                      __uint_as_float(sp.w)};
                float dl[4], dc[4], dd[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = col + 4 * q4 + e;
                    dl[e] = __uint_as_float(r[4 * q4 + e]) * spf[e];
                    dc[e] = -s_sc[j] * dl[e];
                    dd[e] = -s_sc[128 + j] * dl[e];
                }
                pt[2 * q4] = pack2(dl[0], dl[1]);
                pt[2 * q4 + 1] = pack2(dl[2], dl[3]);
                pc[2 * q4] = pack2(dc[0], dc[1]);
                pc[2 * q4 + 1] = pack2(dc[2], dc[3]);
                pd[2 * q4] = pack2(dd[0], dd[1]);
                pd[2 * q4 + 1] = pack2(dd[2], dd[3]);
            }
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const uint32_t o = srow_off(row, col / 8 + h2, 256);
                st_shared_v4(sb + kDt + o, pt[4 * h2], pt[4 * h2 + 1], pt[4 * h2 + 2], pt[4 * h2 + 3]);
                st_shared_v4(sb + kDc + o, pc[4 * h2], pc[4 * h2 + 1], pc[4 * h2 + 2], pc[4 * h2 + 3]);
                st_shared_v4(sb + kDd + o, pd[4 * h2], pd[4 * h2 + 1], pd[4 * h2 + 2], pd[4 * h2 + 3]);
            }
        }
        __syncthreads();
        const size_t ro = (size_t)mt * 128 * 128;
        if (l >= 2) stage_rows_out(sm + kDt, dlt(w, a.o_dlt, l) + ro, 128 * 2, 128, 256);
        stage_rows_out(sm + kDc, dlt(w, a.o_dlc, l) + ro, 128 * 2, 128, 256);
        stage_rows_out(sm + kDd, dlt(w, a.o_dld, l) + ro, 128 * 2, 128, 256);
    };

    for (int c = 0; c < nchunks && ok; ++c) {
        const long t0 = (long)c * a.chunk;
        const int n = (int)min((long)a.chunk, T - t0);
        if (!DBG(n >= 1 && n <= kNmax)) break;  // the same outcome in every CTA

        // ================= forward layers (F_1 also runs the gate scan of every unit)
        for (int l = 1; l < L && ok; ++l) {
            const int per = 2 * HT + (l == 1 ? 1 : 0);
            for (int tile = blockIdx.x; tile < units * per && ok; tile += gridDim.x) {
                const int u = tile / per, lt = tile % per;
                uint8_t* w = unit_ws(u);
                tc_fence_before();
                __syncthreads();
                if (lt == 2 * HT) {
                    // Gate scan of the chunk on one warp (division-free suffix scan), 4 tokens per lane.
                    float* s_g = reinterpret_cast<float*>(sm);  // alpha, eta, theta [3][128]
                    float* s_c = s_g + 3 * kNmax;               // c[128], d[128], A, E, sigma
                    for (int i = tid; i < 3 * kNmax; i += kThreads) {
                        const int which = i / kNmax, j = i % kNmax;
                        const float* g = which == 0 ? a.alpha : (which == 1 ? a.eta : a.theta);
                        const long gi = (long)u * a.gate_ld + (a.chunk_gates ? t0 / a.chunk : t0 + j);
                        const bool in = j < n && DBG(gi < (long)(u + 1) * a.gate_ld);
                        s_g[i] = in ? __ldg(g + gi) : 0.f;
                    }
                    __syncthreads();
                    if (warp == 0) {
                        //   P_j = prod_{l>j} (1 - alpha_l), Q_j = prod_{l>j} eta_l, r_j = P_j + eta_{j+1} r_{j+1}
                        const float* al = s_g;
                        const float* et = s_g + kNmax;
                        const float* th = s_g + 2 * kNmax;
                        float om[4], e4[4], t4[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int j = 4 * lane + i;
                            const bool vj = j < n;
                            om[i] = vj ? 1.f - al[j] : 1.f;
                            e4[i] = vj ? et[j] : 1.f;
                            t4[i] = vj ? th[j] : 0.f;
                        }
                        float ps = om[0] * om[1] * om[2] * om[3], qs = e4[0] * e4[1] * e4[2] * e4[3];
#pragma unroll
                        for (int off = 1; off < 32; off <<= 1) {
                            const float p2 = __shfl_down_sync(0xffffffffu, ps, off);
                            const float q2 = __shfl_down_sync(0xffffffffu, qs, off);
                            if (lane + off < 32) {
                                ps *= p2;
                                qs *= q2;
                            }
                        }
                        float P[4], Q[4];
                        P[3] = __shfl_down_sync(0xffffffffu, ps, 1);
                        Q[3] = __shfl_down_sync(0xffffffffu, qs, 1);
                        if (lane == 31) P[3] = Q[3] = 1.f;
#pragma unroll
                        for (int i = 2; i >= 0; --i) {
                            P[i] = P[i + 1] * om[i + 1];
                            Q[i] = Q[i + 1] * e4[i + 1];
                        }
                        const float e_next = __shfl_down_sync(0xffffffffu, e4[0], 1);
                        float av[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int j = 4 * lane + i;
                            av[i] = j + 1 < n ? (i < 3 ? e4[i + 1] : e_next) : 0.f;
                        }
                        float A = 1.f, B = 0.f;
#pragma unroll
                        for (int i = 3; i >= 0; --i) {
                            B = fmaf(av[i], B, P[i]);
                            A *= av[i];
                        }
#pragma unroll
                        for (int off = 1; off < 32; off <<= 1) {
                            const float A2 = __shfl_down_sync(0xffffffffu, A, off);
                            const float B2 = __shfl_down_sync(0xffffffffu, B, off);
                            if (lane + off < 32) {
                                B = fmaf(A, B2, B);
                                A *= A2;
                            }
                        }
                        float x = __shfl_down_sync(0xffffffffu, B, 1);
                        if (lane == 31) x = 0.f;
                        float r[4];
#pragma unroll
                        for (int i = 3; i >= 0; --i) {
                            x = fmaf(av[i], x, P[i]);
                            r[i] = x;
                        }
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            s_c[4 * lane + i] = t4[i] * r[i];
                            s_c[128 + 4 * lane + i] = t4[i] * Q[i];
                        }
                        if (lane == 0) {
                            s_c[256] = ps;            // A = prod (1 - alpha)
                            s_c[257] = qs;            // E = prod eta
                            s_c[258] = e4[0] * r[0];  // sigma = eta_0 r_0
                        }
                    }
                    __syncthreads();
                    float* gsc = reinterpret_cast<float*>(w + a.o_sc);
                    for (int i = tid; i < 259; i += kThreads) __stcg(gsc + i, s_c[i]);
                    continue;
                }
                const int mt = lt >> 1, p = lt & 1;  // 128 rows of layer l; p 0: keys, 1: queries
                const int K = l == 1 ? D : H;
                for (int k0 = 0; k0 < K; k0 += kKc) {
                    const int kc = min(kKc, K - k0);
                    if (k0 > 0) {
                        tc_fence_before();
                        __syncthreads();
                    }
                    load_kmajor(sb, wb(w, l) + (size_t)mt * 128 * K, K, 128, 128, k0, kc);
                    if (l == 1)
                        load_kmajor(sb + 65536, (p ? a.q : a.k) + ((long)u * T + t0) * D, D, 128, n, k0, kc);
                    else
                        load_mnmajor(sb + 65536, act(w, l - 1) + p * 128, 256, 128, k0, kc, K);
                    operands_ready();
                    if (tid == 0) mma_steps(tmem, sb, false, sb + 65536, l > 1, 128, kc / 16, k0 > 0);
                    if (!mma_done()) {
                        ok = false;
                        break;
                    }
                }
                if (!ok) break;
                forward_epilogue(w, l, mt, p);
            }
            if (!sync() || !ok) {
                ok = false;
                break;
            }
        }
        if (!ok) break;

        // ================= OUT: Y = A_{L-1} W_L^T (unit, keys | queries, 64 output columns)
        {
            const int per = 2 * (D / 64);
            for (int tile = blockIdx.x; tile < units * per && ok; tile += gridDim.x) {
                const int u = tile / per, lt = tile % per, p = lt / (D / 64), nh = lt % (D / 64);
                uint8_t* w = unit_ws(u);
                tc_fence_before();
                __syncthreads();
                load_mnmajor(sb, act(w, L - 1) + p * 128, 256, 128, 0, H, H);
                load_kmajor(sb + 131072, wb(w, L) + (size_t)nh * 64 * H, H, 64, 64, 0, H);
                const __nv_bfloat16* ein = p == 0 ? a.v : a.attn;
                if (ein) stage_rows_in(sb + kInS, ein + ((long)u * T + t0) * D + nh * 64, (size_t)D * 2, n, 128);
                operands_ready();
                if (tid == 0) mma_steps(tmem, sb, true, sb + 131072, false, 64, H / 16, false);
                if (!mma_done()) {
                    ok = false;
                    break;
                }
                float yv[32];
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    uint32_t r[16];
                    tmem_ld16(tmem + lane_off + 32 * half + 16 * b, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) yv[16 * b + i] = __uint_as_float(r[i]);
                }
                constexpr uint32_t kG = 0;
                if (p == 0) {
                    const float* gsc = reinterpret_cast<const float*>(w + a.o_sc);
                    const float cr = -__ldcg(gsc + row), dr = -__ldcg(gsc + 128 + row);
                    const bool valid = row < n;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint32_t og[4] = {0, 0, 0, 0}, oc[4] = {0, 0, 0, 0}, od[4] = {0, 0, 0, 0};
                        if (valid) {
                            const uint4 vv = ld_shared_v4(sb + kInS + srow_off(row, 4 * half + q4, 128));
                            const uint32_t vin[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 vf = unpack_bf16x2(vin[e]);
                                const float g0 = 2.f * (yv[8 * q4 + 2 * e] - vf.x);
                                const float g1 = 2.f * (yv[8 * q4 + 2 * e + 1] - vf.y);
                                og[e] = pack2(g0, g1);
                                oc[e] = pack2(cr * g0, cr * g1);
                                od[e] = pack2(dr * g0, dr * g1);
                            }
                        }
                        const uint32_t o = srow_off(row, 4 * half + q4, 128);
                        st_shared_v4(sb + kG + o, og[0], og[1], og[2], og[3]);
                        st_shared_v4(sb + kG + 16384 + o, oc[0], oc[1], oc[2], oc[3]);
                        st_shared_v4(sb + kG + 32768 + o, od[0], od[1], od[2], od[3]);
                    }
                    __syncthreads();
                    stage_rows_out(sm + kG, w + a.o_gg + nh * 64 * 2, (size_t)D * 2, 128, 128);
                    stage_rows_out(sm + kG + 16384, w + a.o_gc + nh * 64 * 2, (size_t)D * 2, 128, 128);
                    stage_rows_out(sm + kG + 32768, w + a.o_gd + nh * 64 * 2, (size_t)D * 2, 128, 128);
                } else {
                    if (row < n && DBG(t0 + row < T)) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint32_t o[4];
                            uint4 av = make_uint4(0, 0, 0, 0);
                            if (a.attn) av = ld_shared_v4(sb + kInS + srow_off(row, 4 * half + q4, 128));
                            const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float y0 = yv[8 * q4 + 2 * e], y1 = yv[8 * q4 + 2 * e + 1];
                                if (a.attn) {  // memory-as-a-gate output attn * sigmoid(y) (walk-through sec. 4.2)
                                    const float2 a2 = unpack_bf16x2(aw[e]);
                                    y0 = a2.x * fmaf(0.5f, tanh_approx(0.5f * y0), 0.5f);
                                    y1 = a2.y * fmaf(0.5f, tanh_approx(0.5f * y1), 0.5f);
                                }
                                o[e] = pack2(y0, y1);
                            }
                            st_shared_v4(sb + kG + srow_off(row, 4 * half + q4, 128), o[0], o[1], o[2], o[3]);
                        }
                    }
                    __syncthreads();
                    stage_rows_out(sm + kG, a.y + ((long)u * T + t0) * D + nh * 64, (size_t)D * 2, n, 128);
                }
            }
            if (!sync() || !ok) {
                ok = false;
                break;
            }
        }

        // ================= back-propagation: Delta_{L-1} from G, then Delta_{l-1} from Delta_l
        for (int l = L; l >= 2 && ok; --l) {
            for (int tile = blockIdx.x; tile < units * HT && ok; tile += gridDim.x) {
                const int u = tile / HT, mt = tile % HT;  // 128 rows of layer l - 1's output
                uint8_t* w = unit_ws(u);
                tc_fence_before();
                __syncthreads();
                stage_rows_in(sb + kSpS, spp(w, l - 1) + (size_t)mt * 128 * 128, 128 * 4, 128, 512);
                stage_rows_in(sb + kScS, w + a.o_sc, 1024, 1, 1024);  // c[128], d[128]
                const int K = l == L ? D : H;  // the rows of W_l
                for (int k0 = 0; k0 < K; k0 += kKc) {
                    const int kc = min(kKc, K - k0);
                    if (k0 > 0) {
                        tc_fence_before();
                        __syncthreads();
                    }
                    // A = W_l^T rows [mt*128, +128) (MN-major from W_l [out][in]); B = G (K-major) or
                    // Delta_l (MN-major from Delta_l^T [out][tok]).
                    load_mnmajor(sb, wb(w, l) + mt * 128, H, 128, k0, kc, K);
                    if (l == L)
                        load_kmajor(sb + 65536, reinterpret_cast<const __nv_bfloat16*>(w + a.o_gg), D, 128, 128, k0, kc);
                    else
                        load_mnmajor(sb + 65536, dlt(w, a.o_dlt, l), 128, 128, k0, kc, K);
                    operands_ready();
                    if (tid == 0) mma_steps(tmem, sb, true, sb + 65536, l < L, 128, kc / 16, k0 > 0);
                    if (!mma_done()) {
                        ok = false;
                        break;
                    }
                }
                if (!ok) break;
                backprop_epilogue(w, l - 1, mt);
            }
            if (!sync() || !ok) {
                ok = false;
                break;
            }
        }
        if (!ok) break;

        // ================= WGT: weight GEMMs and the state update of every layer
        {
            const int per = 2 * HT + (L - 2) * HT * HT;
            for (int tile = blockIdx.x; tile < units * per && ok; tile += gridDim.x) {
                const int u = tile / per, lt = tile % per;
                uint8_t* w = unit_ws(u);
                int l, mt, nt = 0;
                if (lt < HT) {
                    l = 1;
                    mt = lt;
                } else if (lt < HT + (L - 2) * HT * HT) {
                    const int i = lt - HT;
                    l = 2 + i / (HT * HT);
                    mt = (i % (HT * HT)) / HT;
                    nt = i % HT;
                } else {
                    l = L;
                    mt = lt - HT - (L - 2) * HT * HT;
                }
                const bool last = l == L;
                const int in = l == 1 ? D : H;
                const int N = l == 1 || last ? D : 128;  // accumulator columns
                tc_fence_before();
                __syncthreads();
                if (!last) {
                    // dW_{l,c|d} rows [mt*128, +128) x columns [nt*128, +N) = Delta_l^T diag(-c|-d) A_{l-1}
                    load_kmajor(sb, dlt(w, a.o_dlc, l) + (size_t)mt * 128 * 128, 128, 128, 128, 0, 128);
                    load_kmajor(sb + 32768, dlt(w, a.o_dld, l) + (size_t)mt * 128 * 128, 128, 128, 128, 0, 128);
                    if (l == 1)
                        load_mnmajor(sb + 65536, a.k + ((long)u * T + t0) * D, D, D, 0, 128, n);
                    else
                        load_kmajor(sb + 65536, act(w, l - 1) + (size_t)nt * 128 * 256, 256, 128, 128, 0, 128);
                    stage_rows_in(sb + kStageW, a.W + (size_t)u * a.P + woff(a, l) + (size_t)mt * 128 * in + nt * 128,
                                  (size_t)in * 4, 128, N * 4);
                    stage_rows_in(sb + kStageS, a.S + (size_t)u * a.P + woff(a, l) + (size_t)mt * 128 * in + nt * 128,
                                  (size_t)in * 4, 128, N * 4);
                } else {
                    // dW_{L,c|d}^T rows [mt*128, +128) of the hidden units = A_{L-1} (-c|-d G)
                    load_kmajor(sb, act(w, L - 1) + (size_t)mt * 128 * 256, 256, 128, 128, 0, 128);
                    load_mnmajor(sb + 32768, reinterpret_cast<const __nv_bfloat16*>(w + a.o_gc), D, D, 0, 128, 128);
                    load_mnmajor(sb + 65536, reinterpret_cast<const __nv_bfloat16*>(w + a.o_gd), D, D, 0, 128, 128);
                    // the state tile W_L[0 .. d)[mt*128 .. +128), rows of 512 B
                    stage_rows_in(sb + kStageW, a.W + (size_t)u * a.P + woff(a, L) + mt * 128, (size_t)H * 4, D, 512);
                    stage_rows_in(sb + kStageS, a.S + (size_t)u * a.P + woff(a, L) + mt * 128, (size_t)H * 4, D, 512);
                }
                operands_ready();
                if (tid == 0) {
                    if (!last) {
                        mma_steps(tmem, sb, false, sb + 65536, l == 1, N, 8, false);
                        mma_steps(tmem + 128, sb + 32768, false, sb + 65536, l == 1, N, 8, false);
                    } else {
                        mma_steps(tmem, sb, false, sb + 32768, true, N, 8, false);
                        mma_steps(tmem + 128, sb, false, sb + 65536, true, N, 8, false);
                    }
                }
                if (!mma_done()) {
                    ok = false;
                    break;
                }
                const float* gsc = reinterpret_cast<const float*>(w + a.o_sc);
                const float An = __ldcg(gsc + 256), En = __ldcg(gsc + 257), sig = __ldcg(gsc + 258);
                constexpr uint32_t kWb = 0;  // bf16 rows of the updated weights
                if (!last) {
                    // W <- A W + sigma S + dW_c, S <- E S + dW_d for this thread's row, columns
                    // [half * N/2, +N/2) in blocks of 16
#pragma unroll 1
                    for (int blk = 0; blk < N / 32; ++blk) {
                        const int col = half * (N / 2) + 16 * blk;
                        uint32_t rc[16], rd[16];
                        tmem_ld16(tmem + lane_off + col, rc);
                        tmem_ld16(tmem + lane_off + 128 + col, rd);
                        tmem_wait_ld();
                        uint32_t pk[8];
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const uint32_t o = srow_off(row, col / 4 + q4, N * 4);
                            const float4 wv = *reinterpret_cast<const float4*>(sm + kStageW + o);
                            const float4 sv = *reinterpret_cast<const float4*>(sm + kStageS + o);
                            float wn[4] = {wv.x, wv.y, wv.z, wv.w}, sn[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float wo = wn[e], so = sn[e];
                                wn[e] = fmaf(An, wo, sig * so) + __uint_as_float(rc[4 * q4 + e]);
                                sn[e] = fmaf(En, so, __uint_as_float(rd[4 * q4 + e]));
                            }
                            *reinterpret_cast<float4*>(sm + kStageW + o) = make_float4(wn[0], wn[1], wn[2], wn[3]);
                            *reinterpret_cast<float4*>(sm + kStageS + o) = make_float4(sn[0], sn[1], sn[2], sn[3]);
                            pk[2 * q4] = pack2(wn[0], wn[1]);
                            pk[2 * q4 + 1] = pack2(wn[2], wn[3]);
                        }
                        st_shared_v4(sb + kWb + srow_off(row, col / 8, N * 2), pk[0], pk[1], pk[2], pk[3]);
                        st_shared_v4(sb + kWb + srow_off(row, col / 8 + 1, N * 2), pk[4], pk[5], pk[6], pk[7]);
                    }
                    __syncthreads();
                    const size_t e0 = woff(a, l) + (size_t)mt * 128 * in + nt * 128;
                    stage_rows_out(sm + kWb, wb(w, 1) + e0, (size_t)in * 2, 128, N * 2);
                    stage_rows_out(sm + kStageW, a.W + (size_t)u * a.P + e0, (size_t)in * 4, 128, N * 4);
                    stage_rows_out(sm + kStageS, a.S + (size_t)u * a.P + e0, (size_t)in * 4, 128, N * 4);
                } else {
                    // Transposed tile: this thread's hidden unit j = mt*128 + row, output rows d of W_L.
#pragma unroll 1
                    for (int blk = 0; blk < D / 32; ++blk) {
                        const int d0 = half * (D / 2) + 16 * blk;
                        uint32_t rc[16], rd[16];
                        tmem_ld16(tmem + lane_off + d0, rc);
                        tmem_ld16(tmem + lane_off + 128 + d0, rd);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int d = d0 + e;
                            const uint32_t o = srow_off(d, row >> 2, 512) + 4 * (row & 3);
                            float* pw = reinterpret_cast<float*>(sm + kStageW + o);
                            float* ps = reinterpret_cast<float*>(sm + kStageS + o);
                            const float wo = *pw, so = *ps;
                            const float wn = fmaf(An, wo, sig * so) + __uint_as_float(rc[e]);
                            *pw = wn;
                            *ps = fmaf(En, so, __uint_as_float(rd[e]));
                            *reinterpret_cast<__nv_bfloat16*>(sm + kWb + srow_off(d, row >> 3, 256) + 2 * (row & 7)) =
                                __float2bfloat16_rn(wn);
                        }
                    }
                    __syncthreads();
                    const size_t e0 = woff(a, L) + mt * 128;
                    stage_rows_out(sm + kWb, wb(w, 1) + e0, (size_t)H * 2, D, 256);
                    stage_rows_out(sm + kStageW, a.W + (size_t)u * a.P + e0, (size_t)H * 4, D, 512);
                    stage_rows_out(sm + kStageS, a.S + (size_t)u * a.P + e0, (size_t)H * 4, D, 512);
                }
            }
            if (!sync() || !ok) {
                ok = false;
                break;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

#undef DBG

size_t tc_deep_ws_bytes_per_unit(int d, int h, int layers) {
    DeepTcArgs a{};
    return deep_layout(d, h, layers, a);
}

bool tc_deep_supported(int d, int h, int layers, int chunk) {
    return (d == 64 || d == 128) && h == 4 * d && layers >= 3 && layers <= 8 && chunk >= 1 && chunk <= dp::kNmax;
}

cudaError_t launch_chunk_tc_deep(const ForwardArgs& f, int layers, unsigned* sync, cudaStream_t st) {
    if (!f.bf16 || !tc_deep_supported(f.d, f.h, layers, f.chunk)) return cudaErrorInvalidValue;
    static std::atomic<unsigned> attr_set{0};
    static std::atomic<int> sm_count[32];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 32) return cudaErrorInvalidDevice;
    const unsigned bit = 1u << dev;
    if (!(attr_set.load() & bit)) {
        e = cudaFuncSetAttribute(chunk_fwd_tc_deep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dp::kSmemBytes);
        if (e != cudaSuccess) return e;
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chunk_fwd_tc_deep, dp::kThreads, dp::kSmemBytes);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        sm_count[dev].store(sms);
        attr_set.fetch_or(bit);
    }
    DeepTcArgs a{};
    const size_t need = deep_layout(f.d, f.h, layers, a);
    if (f.ws_per_unit * sizeof(float) < need) return cudaErrorInvalidValue;
    a.k = (const __nv_bfloat16*)f.k;
    a.q = (const __nv_bfloat16*)f.q;
    a.v = (const __nv_bfloat16*)f.v;
    a.alpha = f.alpha;
    a.eta = f.eta;
    a.theta = f.theta;
    a.W = f.W1;
    a.S = f.S1;
    a.y = (__nv_bfloat16*)f.y;
    a.attn = (const __nv_bfloat16*)f.attn;
    a.ws = reinterpret_cast<uint8_t*>(f.ws);
    a.ws_stride = f.ws_per_unit * sizeof(float);
    a.T = f.T;
    a.gate_ld = f.gate_ld;
    a.P = (long)2 * f.d * f.h + (long)(layers - 2) * f.h * f.h;
    a.chunk = f.chunk;
    a.units = (int)f.units;
    a.D = f.d;
    a.H = f.h;
    a.L = layers;
    a.chunk_gates = f.chunk_gates ? 1 : 0;
    a.status = f.status;
    a.sync = sync;
    e = cudaMemsetAsync(sync, 0, 2 * sizeof(unsigned), st);
    if (e != cudaSuccess) return e;
    void* params[] = {&a};
    return cudaLaunchCooperativeKernel((const void*)chunk_fwd_tc_deep, dim3((unsigned)sm_count[dev].load()),
                                       dim3(dp::kThreads), params, dp::kSmemBytes, st);
}

}  // namespace titans
