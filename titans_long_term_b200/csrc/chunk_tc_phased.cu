// Tensor-core chunk forward for the wide MLP memory M(x) = W2 silu(W1 x), d = 128, h = 512,
// chunk n <= 128, bf16 operands with fp32 accumulation, fp32 state.
//
// Method ("Titans: Learning to Memorize at Test Time", walk-through sec. 3.1-3.2): every token of
// a chunk takes its gradient of ||M(k) - v||^2 at the chunk-start weights, so the chunk's momentum
// and forgetting recurrence folds into
//   W <- A W + sigma S - sum_j c_j g_j,   S <- E S - sum_j d_j g_j,
// with c_j, d_j, A, E, sigma from a division-free suffix scan of the gates, and the sums of
// per-token outer products are weighted GEMMs.
//
// One unit's state is 1 MiB of fp32 (W1, S1 [512 x 128], W2, S2 [128 x 512]): it does not fit
// one SM, so this kernel does not keep it on chip. Instead one persistent CTA per SM walks the
// chunks of every unit together in four phases, each a set of 128-row tcgen05 tiles spread over
// all SMs, separated by grid-wide barriers:
//   P1  Z^T [h x tok] = W1 [K; Q]^T (128 hidden rows x 128 tokens per tile) -> silu(Z)^T (bf16)
//       and silu'(Z_K)^T (fp32); plus, per unit, the gate scan and the scaled key tiles -c K, -d K.
//   P2  Y [tok x d] = silu(Z) W2^T (128 tokens x 64 columns per tile) -> keys: G = 2 (Y - v) and
//       its scaled copies -c G, -d G (bf16, each rounded once from fp32); queries: y (or the
//       gated output attn * sigmoid(y)).
//   P3  (GW2)^T [h x tok] = W2^T G^T -> Delta^T = (GW2)^T * silu'(Z_K)^T (bf16).
//   P4  dW1_{c,d} [h x d] = Delta^T diag(-c|-d) K and dW2_{c,d} [d x h] = G^T diag(-c|-d) silu(Z_K),
//       two TMEM accumulators per tile; the epilogue applies W <- A W + sigma S + dW_c,
//       S <- E S + dW_d in fp32 and rewrites the bf16 copy of W that the next chunk's MMAs read.
// The state and the intermediates (about 1 MiB per unit each) stay in L2 between phases. Operand
// tiles are copied into shared memory with cp.async in the 128-byte swizzled layout the MMA
// descriptors describe; one thread issues the MMAs, fp32 accumulators live in TMEM, and every
// thread reads its own TMEM row in the epilogue.
//
// The grid barrier spins on a global counter with a 1 s bound; a timeout sets the device status
// word and a global abort flag that every other CTA sees in its own spin, so all CTAs leave.
// The kernel is launched cooperatively, which guarantees that all CTAs are resident together.
#include <cuda_bf16.h>

#include <atomic>
#include <cstdint>

#include "kernels.h"
#include "phased_common.cuh"
#include "ptx.cuh"

namespace titans {

namespace ph {
constexpr int kD = 128, kH = 512, kNmax = 128;
using phc::kThreads;
// Per-unit workspace (bytes), each piece 1024-aligned.
constexpr size_t W1B = 0;                                  // bf16 [h][d]   copy of W1
constexpr size_t W2B = W1B + (size_t)kH * kD * 2;          // bf16 [d][h]   copy of W2
constexpr size_t AT = W2B + (size_t)kD * kH * 2;           // bf16 [h][2 x 128 tok]  silu(Z)^T: keys, then queries
constexpr size_t SP = AT + (size_t)kH * 256 * 2;           // fp32 [h][128 tok]      silu'(Z_K)^T
constexpr size_t DT = SP + (size_t)kH * kNmax * 4;         // bf16 [h][128 tok]      Delta^T
constexpr size_t GG = DT + (size_t)kH * kNmax * 2;         // bf16 [128 tok][d]      G
constexpr size_t GC = GG + (size_t)kNmax * kD * 2;         // bf16 [128 tok][d]      -c G
constexpr size_t GD = GC + (size_t)kNmax * kD * 2;         // bf16 [128 tok][d]      -d G
constexpr size_t KC = GD + (size_t)kNmax * kD * 2;         // bf16 [128 tok][d]      -c K
constexpr size_t KD = KC + (size_t)kNmax * kD * 2;         // bf16 [128 tok][d]      -d K
constexpr size_t SC = KD + (size_t)kNmax * kD * 2;         // fp32 c[128], d[128], A, E, sigma
constexpr size_t kWsBytes = SC + 2048;
// Shared memory: operand tiles, each [rows][64] bf16 with the 128-byte swizzle.
constexpr uint32_t kSmemOperands = 224 * 1024;
// P4 stages the fp32 W and S tiles it updates ([128 rows][128 floats] each) after its 96 KB of
// MMA operands.
constexpr uint32_t kStageW = 96 * 1024, kStageS = 160 * 1024;
// Epilogue staging (row-contiguous copies out): in the operand area, free once a tile's MMAs
// completed, except for inputs staged with the operands.
constexpr uint32_t kP1At = 0, kP1Sp = 32 * 1024;    // silu(Z)^T [128][256 B], silu'(Z_K)^T [128][512 B]
constexpr uint32_t kP2G = 0, kP2In = 192 * 1024;    // G, -cG, -dG (or y) [128][128 B] each; v or attn [128][128 B]
constexpr uint32_t kP3Dt = 0, kP3Sp = 64 * 1024;    // Delta^T [128][256 B]; silu'(Z_K)^T rows [128][512 B]
constexpr uint32_t kP4Wb = 0;                       // bf16 weight rows [128][256 B]
constexpr uint32_t BAR = kSmemOperands;       // one mbarrier (MMA completion)
constexpr uint32_t TPTR = BAR + 8;
constexpr uint32_t OKF = TPTR + 4;            // the grid barrier's outcome for the CTA
constexpr uint32_t END = OKF + 4;
constexpr size_t kSmemBytes = END + 1024;
constexpr uint32_t kTmemCols = 256;
}  // namespace ph

static_assert(ph::kSmemBytes <= 232448, "shared memory budget");

struct PhasedArgs {
    const __nv_bfloat16 *k, *q, *v;
    const float *alpha, *eta, *theta;
    float *W1, *W2, *S1, *S2;
    __nv_bfloat16* y;
    const __nv_bfloat16* attn;
    uint8_t* ws;
    size_t ws_stride;  // bytes per unit
    long T, gate_ld;
    int chunk, units;
    int chunk_gates;   // gates shared by a chunk's tokens ([units][chunks]) instead of per token
    unsigned* status;
    unsigned* sync;    // [0] barrier arrivals, [1] abort flag; zero at launch
};

namespace {
using phc::load_tile;
using phc::operands_ready;
using phc::pack2;
using phc::srow_off;
using phc::stage_in;
using phc::stage_off;
using phc::stage_rows_in;
using phc::stage_rows_out;
using phc::tanh_approx;

__device__ __forceinline__ bool grid_sync(const PhasedArgs& a, unsigned& epoch, volatile uint32_t* s_ok) {
    return phc::grid_sync(a.sync, a.status, epoch, s_ok);
}

}  // namespace

__global__ void __launch_bounds__(ph::kThreads, 1) chunk_fwd_tc_phased(const __grid_constant__ PhasedArgs a) {
    using namespace ph;
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

    // Issue on one thread, wait on all: the tile's MMAs are complete and TMEM is readable. The
    // outcome is the same for every thread of the CTA (a timeout anywhere counts for all).
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
    auto unit_ws = [&](int u) { return a.ws + (size_t)u * a.ws_stride; };
#define DBG(cond) TITANS_DBG(cond, a.status, reinterpret_cast<volatile int*>(&a.sync[1]))

    const int units = a.units;
    const long T = a.T;
    const int nchunks = (int)((T + a.chunk - 1) / a.chunk);
    // every workspace piece of a unit lies inside its stride; a chunk fits the 128-token tiles
    if (!DBG(a.ws_stride >= kWsBytes && a.chunk >= 1 && a.chunk <= kNmax)) ok = false;

    // ---- prologue: bf16 copies of the initial weights
    for (long i = (long)blockIdx.x * kThreads + tid; i < (long)units * kH * kD / 4; i += (long)gridDim.x * kThreads) {
        const long e = 4 * i;
        const int u = (int)(e / (kH * kD));
        const long r = e % (kH * kD);
        const float4 w1 = __ldcg(reinterpret_cast<const float4*>(a.W1 + e));
        const float4 w2 = __ldcg(reinterpret_cast<const float4*>(a.W2 + e));
        uint2* d1 = reinterpret_cast<uint2*>(unit_ws(u) + W1B + 2 * r);
        uint2* d2 = reinterpret_cast<uint2*>(unit_ws(u) + W2B + 2 * r);
        __stcg(d1, make_uint2(pack2(w1.x, w1.y), pack2(w1.z, w1.w)));
        __stcg(d2, make_uint2(pack2(w2.x, w2.y), pack2(w2.z, w2.w)));
    }
    ok = grid_sync(a, epoch, s_ok) && ok;

    for (int c = 0; c < nchunks && ok; ++c) {
        const long t0 = (long)c * a.chunk;
        const int n = (int)min((long)a.chunk, T - t0);
        if (!DBG(n >= 1 && n <= kNmax)) break;  // the same outcome in every CTA

        // ================= P1: Z^T tiles (unit, 128 hidden rows, keys | queries) and gate scans
        const int p1_gemm = units * 8;
        for (int tile = blockIdx.x; tile < p1_gemm + units && ok; tile += gridDim.x) {
            if (tile >= p1_gemm) {
                // Gate scan of the chunk (sequential suffix scan, division-free) and the scaled keys.
                const int u = tile - p1_gemm;
                uint8_t* w = unit_ws(u);
                float* s_c = reinterpret_cast<float*>(sm);  // shared scratch: c[128], d[128], A, E, sigma
                float* s_d = s_c + 128;
                float* s_g = s_c + 512;                     // the chunk's gates: alpha, eta, theta [3][128]
                for (int i = tid; i < 3 * kNmax; i += kThreads) {
                    const int which = i / kNmax, j = i % kNmax;
                    const float* g = which == 0 ? a.alpha : (which == 1 ? a.eta : a.theta);
                    const long gi = (long)u * a.gate_ld + (a.chunk_gates ? t0 / a.chunk : t0 + j);
                    const bool in = j < n && DBG(gi < (long)(u + 1) * a.gate_ld);
                    s_g[i] = in ? __ldg(g + gi) : 0.f;
                }
                __syncthreads();
                if (warp == 0) {
                    // The suffix scan on one warp, tokens j = 4 lane + i (gates past n are neutral):
                    //   P_j = prod_{l>j} (1 - alpha_l), Q_j = prod_{l>j} eta_l, r_j = P_j + eta_{j+1} r_{j+1}
                    // with the chain cut after the last token; products and the affine maps of r are
                    // combined across lanes with shuffles.
                    const float* al = s_g;
                    const float* et = s_g + kNmax;
                    const float* th = s_g + 2 * kNmax;
                    float om[4], e4[4], t4[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int j = 4 * lane + i;
                        const bool v = j < n;
                        om[i] = v ? 1.f - al[j] : 1.f;
                        e4[i] = v ? et[j] : 1.f;
                        t4[i] = v ? th[j] : 0.f;
                    }
                    float ps = om[0] * om[1] * om[2] * om[3], qs = e4[0] * e4[1] * e4[2] * e4[3];
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {  // inclusive suffix products over lanes
                        const float p2 = __shfl_down_sync(0xffffffffu, ps, off), q2 = __shfl_down_sync(0xffffffffu, qs, off);
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
                    // r_j = a_j r_{j+1} + P_j, a_j = eta_{j+1} while j + 1 < n, else 0
                    const float e_next = __shfl_down_sync(0xffffffffu, e4[0], 1);
                    float av[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int j = 4 * lane + i;
                        av[i] = j + 1 < n ? (i < 3 ? e4[i + 1] : e_next) : 0.f;
                    }
                    float A = 1.f, B = 0.f;  // this lane's map r_{4 lane} = A r_{4 lane + 4} + B
#pragma unroll
                    for (int i = 3; i >= 0; --i) {
                        B = fmaf(av[i], B, P[i]);
                        A *= av[i];
                    }
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const float A2 = __shfl_down_sync(0xffffffffu, A, off), B2 = __shfl_down_sync(0xffffffffu, B, off);
                        if (lane + off < 32) {
                            B = fmaf(A, B2, B);
                            A *= A2;
                        }
                    }
                    float x = __shfl_down_sync(0xffffffffu, B, 1);  // r of the next lane's first token
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
                        s_d[4 * lane + i] = t4[i] * Q[i];
                    }
                    if (lane == 0) {
                        s_c[256] = ps;            // A = prod (1 - alpha)
                        s_c[257] = qs;            // E = prod eta
                        s_c[258] = e4[0] * r[0];  // sigma = eta_0 r_0
                    }
                }
                __syncthreads();
                float* gsc = reinterpret_cast<float*>(w + SC);
                for (int i = tid; i < 259; i += kThreads) __stcg(gsc + i, s_c[i]);
                // -c_j K_j and -d_j K_j, bf16 [128 tok][d]; rows j >= n are zero
                const __nv_bfloat16* K = a.k + ((long)u * T + t0) * kD;
                for (int i = tid; i < kNmax * kD / 8; i += kThreads) {
                    const int j = i / (kD / 8), c8 = i % (kD / 8);
                    uint4 oc = make_uint4(0, 0, 0, 0), od = oc;
                    if (j < n) {
                        const uint4 kv = __ldg(reinterpret_cast<const uint4*>(K + (long)j * kD) + c8);
                        const uint32_t kin[4] = {kv.x, kv.y, kv.z, kv.w};
                        uint32_t pc[4], pd[4];
                        const float cj = -s_c[j], dj = -s_d[j];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = unpack_bf16x2(kin[e]);
                            pc[e] = pack2(cj * f.x, cj * f.y);
                            pd[e] = pack2(dj * f.x, dj * f.y);
                        }
                        oc = make_uint4(pc[0], pc[1], pc[2], pc[3]);
                        od = make_uint4(pd[0], pd[1], pd[2], pd[3]);
                    }
                    __stcg(reinterpret_cast<uint4*>(w + KC) + i, oc);
                    __stcg(reinterpret_cast<uint4*>(w + KD) + i, od);
                }
                __syncthreads();
                continue;
            }
            const int u = tile >> 3, mt = (tile >> 1) & 3, part = tile & 1;  // part 0: keys, 1: queries
            uint8_t* w = unit_ws(u);
            const __nv_bfloat16* X = (part ? a.q : a.k) + ((long)u * T + t0) * kD;
            // A = W1 rows [mt*128, +128) (K-major, two 64-column blocks), B = the chunk's tokens.
            tc_fence_before();
            __syncthreads();
            for (int kb = 0; kb < 2; ++kb) {
                load_tile(sb + kb * 16384, w + W1B + ((size_t)mt * 128 * kD + kb * 64) * 2, kD * 2, 128, 128);
                load_tile(sb + 32768 + kb * 16384, reinterpret_cast<const uint8_t*>(X + kb * 64), kD * 2, 128, n);
            }
            operands_ready();
            if (tid == 0) {
                const uint32_t id = idesc_bf16_f32(128, 128, 0, 0);
                for (int kb = 0; kb < 2; ++kb)
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(tmem, sdesc_sw128(sb + kb * 16384 + ks * 32, 16, 1024),
                                  sdesc_sw128(sb + 32768 + kb * 16384 + ks * 32, 16, 1024), id, (kb | ks) != 0);
            }
            if (!mma_done()) {
                ok = false;
                break;
            }
            // Epilogue: hidden row mt*128 + row, tokens [64 half, +64). The outputs are staged in the
            // operand area (free once the MMAs completed) and copied out row-contiguously.
#pragma unroll 1
            for (int blk = 0; blk < 4; ++blk) {
                uint32_t r[16];
                tmem_ld16(tmem + lane_off + 64 * half + 16 * blk, r);
                tmem_wait_ld();
                uint32_t pk[8];
                float spv[16];
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    // sigma(z) = (1 + tanh(z / 2)) / 2 (one MUFU op), silu(z) = z sigma(z)
                    const float z0 = __uint_as_float(r[i]), z1 = __uint_as_float(r[i + 1]);
                    const float s0 = fmaf(0.5f, tanh_approx(0.5f * z0), 0.5f);
                    const float s1 = fmaf(0.5f, tanh_approx(0.5f * z1), 0.5f);
                    const float a0 = z0 * s0, a1 = z1 * s1;
                    pk[i / 2] = pack2(a0, a1);
                    spv[i] = s0 + a0 * (1.f - s0);  // silu'(z) = sigma + silu (1 - sigma)
                    spv[i + 1] = s1 + a1 * (1.f - s1);
                }
                st_shared_v4(sb + kP1At + srow_off(row, 8 * half + 2 * blk, 256), pk[0], pk[1], pk[2], pk[3]);
                st_shared_v4(sb + kP1At + srow_off(row, 8 * half + 2 * blk + 1, 256), pk[4], pk[5], pk[6], pk[7]);
                if (part == 0) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        st_shared_v4(sb + kP1Sp + srow_off(row, 16 * half + 4 * blk + q4, 512),
                                     __float_as_uint(spv[4 * q4]), __float_as_uint(spv[4 * q4 + 1]),
                                     __float_as_uint(spv[4 * q4 + 2]), __float_as_uint(spv[4 * q4 + 3]));
                }
            }
            __syncthreads();
            stage_rows_out(sm + kP1At, w + AT + ((size_t)mt * 128 * 256 + part * 128) * 2, 256 * 2, 128, 256);
            if (part == 0)
                stage_rows_out(sm + kP1Sp, w + SP + (size_t)mt * 128 * kNmax * 4, kNmax * 4, 128, 512);
        }
        if (!grid_sync(a, epoch, s_ok) || !ok) {
            ok = false;
            break;
        }

        // ================= P2: Y tiles (unit, keys | queries, 64 output columns)
        for (int tile = blockIdx.x; tile < units * 4 && ok; tile += gridDim.x) {
            const int u = tile >> 2, part = (tile >> 1) & 1, nh = tile & 1;
            uint8_t* w = unit_ws(u);
            tc_fence_before();
            __syncthreads();
            // A = silu(Z) [tok x h] from silu(Z)^T (MN-major): per 64-hidden block kb two 64-token
            // blocks 8 KB apart; B = W2 rows [nh*64, +64) (K-major: the hidden index is contiguous).
            for (int kb = 0; kb < 8; ++kb) {
                for (int mb = 0; mb < 2; ++mb)
                    load_tile(sb + kb * 16384 + mb * 8192, w + AT + ((size_t)kb * 64 * 256 + part * 128 + mb * 64) * 2,
                              256 * 2, 64, 64);
                load_tile(sb + 131072 + kb * 8192, w + W2B + ((size_t)nh * 64 * kH + kb * 64) * 2, kH * 2, 64, 64);
            }
            // The epilogue's other input, staged row-contiguously: v (keys) or attn (gated queries),
            // tokens [t0, t0 + n), columns [nh*64, +64).
            const __nv_bfloat16* ein = part == 0 ? a.v : a.attn;
            if (ein) stage_rows_in(sb + kP2In, ein + ((long)u * T + t0) * kD + nh * 64, kD * 2, n, 128);
            operands_ready();
            if (tid == 0) {
                const uint32_t id = idesc_bf16_f32(128, 64, 1, 0);
                for (int kb = 0; kb < 8; ++kb)
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(tmem, sdesc_sw128(sb + kb * 16384 + ks * 2048, 8192, 1024),
                                  sdesc_sw128(sb + 131072 + kb * 8192 + ks * 32, 16, 1024), id, (kb | ks) != 0);
            }
            if (!mma_done()) {
                ok = false;
                break;
            }
            // Epilogue: token row `row`, output columns nh*64 + 32 half + [0, 32).
            float yv[32];
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                uint32_t r[16];
                tmem_ld16(tmem + lane_off + 32 * half + 16 * b, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) yv[16 * b + i] = __uint_as_float(r[i]);
            }
            if (part == 0) {
                const float* gsc = reinterpret_cast<const float*>(w + SC);
                const float cr = -__ldcg(gsc + row), dr = -__ldcg(gsc + 128 + row);
                const bool valid = row < n;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t og[4] = {0, 0, 0, 0}, oc[4] = {0, 0, 0, 0}, od[4] = {0, 0, 0, 0};
                    if (valid) {
                        const uint4 vv = ld_shared_v4(sb + kP2In + srow_off(row, 4 * half + q4, 128));
                        const uint32_t vin[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 vf = unpack_bf16x2(vin[e]);
                            const float g0 = 2.f * (yv[8 * q4 + 2 * e] - vf.x), g1 = 2.f * (yv[8 * q4 + 2 * e + 1] - vf.y);
                            og[e] = pack2(g0, g1);
                            oc[e] = pack2(cr * g0, cr * g1);
                            od[e] = pack2(dr * g0, dr * g1);
                        }
                    }
                    const uint32_t o = srow_off(row, 4 * half + q4, 128);
                    st_shared_v4(sb + kP2G + o, og[0], og[1], og[2], og[3]);
                    st_shared_v4(sb + kP2G + 16384 + o, oc[0], oc[1], oc[2], oc[3]);
                    st_shared_v4(sb + kP2G + 32768 + o, od[0], od[1], od[2], od[3]);
                }
                __syncthreads();
                // rows >= n are zero: they are operands of the next phases
                stage_rows_out(sm + kP2G, w + GG + nh * 64 * 2, kD * 2, 128, 128);
                stage_rows_out(sm + kP2G + 16384, w + GC + nh * 64 * 2, kD * 2, 128, 128);
                stage_rows_out(sm + kP2G + 32768, w + GD + nh * 64 * 2, kD * 2, 128, 128);
            } else {
                if (row < n && DBG(t0 + row < T)) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint32_t o[4];
                        uint4 av = make_uint4(0, 0, 0, 0);
                        if (a.attn) av = ld_shared_v4(sb + kP2In + srow_off(row, 4 * half + q4, 128));
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
                        st_shared_v4(sb + kP2G + srow_off(row, 4 * half + q4, 128), o[0], o[1], o[2], o[3]);
                    }
                }
                __syncthreads();
                stage_rows_out(sm + kP2G, a.y + ((long)u * T + t0) * kD + nh * 64, kD * 2, n, 128);
            }
        }
        if (!grid_sync(a, epoch, s_ok) || !ok) {
            ok = false;
            break;
        }

        // ================= P3: (GW2)^T tiles (unit, 128 hidden rows) -> Delta^T
        for (int tile = blockIdx.x; tile < units * 4 && ok; tile += gridDim.x) {
            const int u = tile >> 2, mt = tile & 3;
            uint8_t* w = unit_ws(u);
            tc_fence_before();
            __syncthreads();
            // A = W2^T rows [mt*128, +128) from W2 [d][h] (MN-major: per 64-column block kb of d, two
            // 64-hidden blocks 8 KB apart); B = G [tok][d] (K-major).
            for (int kb = 0; kb < 2; ++kb) {
                for (int mb = 0; mb < 2; ++mb)
                    load_tile(sb + kb * 16384 + mb * 8192, w + W2B + ((size_t)kb * 64 * kH + mt * 128 + mb * 64) * 2,
                              kH * 2, 64, 64);
                load_tile(sb + 32768 + kb * 16384, w + GG + (size_t)kb * 64 * 2, kD * 2, 128, 128);
            }
            stage_rows_in(sb + kP3Sp, w + SP + (size_t)mt * 128 * kNmax * 4, kNmax * 4, 128, 512);  // silu'(Z_K)^T rows
            operands_ready();
            if (tid == 0) {
                const uint32_t id = idesc_bf16_f32(128, 128, 1, 0);
                for (int kb = 0; kb < 2; ++kb)
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(tmem, sdesc_sw128(sb + kb * 16384 + ks * 2048, 8192, 1024),
                                  sdesc_sw128(sb + 32768 + kb * 16384 + ks * 32, 16, 1024), id, (kb | ks) != 0);
            }
            if (!mma_done()) {
                ok = false;
                break;
            }
#pragma unroll 1
            for (int blk = 0; blk < 4; ++blk) {
                uint32_t r[16];
                tmem_ld16(tmem + lane_off + 64 * half + 16 * blk, r);
                tmem_wait_ld();
                uint32_t pk[8];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint4 sp = ld_shared_v4(sb + kP3Sp + srow_off(row, 16 * half + 4 * blk + q4, 512));
                    pk[2 * q4] = pack2(__uint_as_float(r[4 * q4]) * __uint_as_float(sp.x),
                                       __uint_as_float(r[4 * q4 + 1]) * __uint_as_float(sp.y));
                    pk[2 * q4 + 1] = pack2(__uint_as_float(r[4 * q4 + 2]) * __uint_as_float(sp.z),
                                           __uint_as_float(r[4 * q4 + 3]) * __uint_as_float(sp.w));
                }
                st_shared_v4(sb + kP3Dt + srow_off(row, 8 * half + 2 * blk, 256), pk[0], pk[1], pk[2], pk[3]);
                st_shared_v4(sb + kP3Dt + srow_off(row, 8 * half + 2 * blk + 1, 256), pk[4], pk[5], pk[6], pk[7]);
            }
            __syncthreads();
            stage_rows_out(sm + kP3Dt, w + DT + (size_t)mt * 128 * kNmax * 2, kNmax * 2, 128, 256);
        }
        if (!grid_sync(a, epoch, s_ok) || !ok) {
            ok = false;
            break;
        }

        // ================= P4: weight GEMMs and the state update (unit, W1 | W2, 128-row block)
        for (int tile = blockIdx.x; tile < units * 8 && ok; tile += gridDim.x) {
            const int u = tile >> 3, which = (tile >> 2) & 1, mt = tile & 3;
            uint8_t* w = unit_ws(u);
            tc_fence_before();
            __syncthreads();
            const uint32_t A0 = sb, B0 = sb + 32768, C0 = sb + 65536;  // A | B c-part | B d-part (or A c/d, B)
            if (which == 0) {
                // dW1_{c,d} [h x d] = Delta^T (K-major [h][tok]) x diag(-c|-d) K (MN-major [tok][d]).
                for (int kb = 0; kb < 2; ++kb) {
                    load_tile(A0 + kb * 16384, w + DT + ((size_t)mt * 128 * kNmax + kb * 64) * 2, kNmax * 2, 128, 128);
                    for (int mb = 0; mb < 2; ++mb) {
                        load_tile(B0 + kb * 16384 + mb * 8192, w + KC + ((size_t)kb * 64 * kD + mb * 64) * 2, kD * 2,
                                  64, 64);
                        load_tile(C0 + kb * 16384 + mb * 8192, w + KD + ((size_t)kb * 64 * kD + mb * 64) * 2, kD * 2,
                                  64, 64);
                    }
                }
            } else {
                // dW2_{c,d} [d x h] = (diag(-c|-d) G)^T (MN-major [tok][d]) x silu(Z_K) (K-major [h][tok]).
                for (int kb = 0; kb < 2; ++kb) {
                    for (int mb = 0; mb < 2; ++mb) {
                        load_tile(A0 + kb * 16384 + mb * 8192, w + GC + ((size_t)kb * 64 * kD + mb * 64) * 2, kD * 2,
                                  64, 64);
                        load_tile(C0 + kb * 16384 + mb * 8192, w + GD + ((size_t)kb * 64 * kD + mb * 64) * 2, kD * 2,
                                  64, 64);
                    }
                    load_tile(B0 + kb * 16384, w + AT + ((size_t)mt * 128 * 256 + kb * 64) * 2, 256 * 2, 128, 128);
                }
            }
            // The fp32 rows this tile updates, staged with coalesced copies: W1 rows [mt*128, +128)
            // (one contiguous 64 KB block) or W2 rows 0..127 at hidden columns [mt*128, +128).
            float* Wg;
            float* Sg;
            size_t ldw;
            if (which == 0) {
                Wg = a.W1 + ((size_t)u * kH + mt * 128) * kD;
                Sg = a.S1 + ((size_t)u * kH + mt * 128) * kD;
                ldw = kD;
            } else {
                Wg = a.W2 + (size_t)u * kD * kH + mt * 128;
                Sg = a.S2 + (size_t)u * kD * kH + mt * 128;
                ldw = kH;
            }
            stage_in(sb + kStageW, Wg, ldw);
            stage_in(sb + kStageS, Sg, ldw);
            operands_ready();
            if (tid == 0) {
                for (int kb = 0; kb < 2; ++kb)
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint32_t acc = (kb | ks) != 0;
                        if (which == 0) {
                            const uint32_t id = idesc_bf16_f32(128, 128, 0, 1);
                            const uint64_t da = sdesc_sw128(A0 + kb * 16384 + ks * 32, 16, 1024);
                            umma_bf16(tmem, da, sdesc_sw128(B0 + kb * 16384 + ks * 2048, 8192, 1024), id, acc);
                            umma_bf16(tmem + 128, da, sdesc_sw128(C0 + kb * 16384 + ks * 2048, 8192, 1024), id, acc);
                        } else {
                            const uint32_t id = idesc_bf16_f32(128, 128, 1, 0);
                            const uint64_t db = sdesc_sw128(B0 + kb * 16384 + ks * 32, 16, 1024);
                            umma_bf16(tmem, sdesc_sw128(A0 + kb * 16384 + ks * 2048, 8192, 1024), db, id, acc);
                            umma_bf16(tmem + 128, sdesc_sw128(C0 + kb * 16384 + ks * 2048, 8192, 1024), db, id, acc);
                        }
                    }
            }
            if (!mma_done()) {
                ok = false;
                break;
            }
            // Epilogue: W <- A W + sigma S + dW_c, S <- E S + dW_d for this thread's row of the tile,
            // in place in the staged tiles; then the bf16 copy of the row, and coalesced copies out.
            const float* gsc = reinterpret_cast<const float*>(w + SC);
            const float An = __ldcg(gsc + 256), En = __ldcg(gsc + 257), sig = __ldcg(gsc + 258);
#pragma unroll 1
            for (int blk = 0; blk < 4; ++blk) {
                uint32_t rc[16], rd[16];
                tmem_ld16(tmem + lane_off + 64 * half + 16 * blk, rc);
                tmem_ld16(tmem + lane_off + 128 + 64 * half + 16 * blk, rd);
                tmem_wait_ld();
                uint32_t pk[8];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint32_t o = stage_off(row, 16 * half + 4 * blk + q4);
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
                st_shared_v4(sb + kP4Wb + srow_off(row, 8 * half + 2 * blk, 256), pk[0], pk[1], pk[2], pk[3]);
                st_shared_v4(sb + kP4Wb + srow_off(row, 8 * half + 2 * blk + 1, 256), pk[4], pk[5], pk[6], pk[7]);
            }
            __syncthreads();
            // the bf16 copy of the rows: W1 rows [mt*128, +128) or W2 rows 0..127 at hidden [mt*128, +128)
            if (which == 0)
                stage_rows_out(sm + kP4Wb, w + W1B + (size_t)mt * 128 * kD * 2, kD * 2, 128, 256);
            else
                stage_rows_out(sm + kP4Wb, w + W2B + (size_t)mt * 128 * 2, kH * 2, 128, 256);
            for (int i = tid; i < 128 * 32; i += kThreads) {
                const int r = i >> 5, cc = i & 31;
                const uint32_t o = stage_off(r, cc);
                __stcg(reinterpret_cast<float4*>(Wg + (size_t)r * ldw + 4 * cc),
                       *reinterpret_cast<const float4*>(sm + kStageW + o));
                __stcg(reinterpret_cast<float4*>(Sg + (size_t)r * ldw + 4 * cc),
                       *reinterpret_cast<const float4*>(sm + kStageS + o));
            }
        }
        if (!grid_sync(a, epoch, s_ok) || !ok) {
            ok = false;
            break;
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

size_t tc_phased_ws_bytes_per_unit() { return ph::kWsBytes; }

bool tc_phased_supported(int d, int h, int chunk) { return d == 128 && h == 512 && chunk >= 1 && chunk <= 128; }

cudaError_t launch_chunk_tc_phased(const ForwardArgs& f, unsigned* sync, cudaStream_t st) {
    static std::atomic<unsigned long long> attr_set{0};
    static std::atomic<int> sm_count[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const unsigned long long bit = 1ull << dev;
    if (!(attr_set.load() & bit)) {
        e = cudaFuncSetAttribute(chunk_fwd_tc_phased, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ph::kSmemBytes);
        if (e != cudaSuccess) return e;
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chunk_fwd_tc_phased, ph::kThreads, ph::kSmemBytes);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        sm_count[dev].store(sms);
        attr_set.fetch_or(bit);
    }
    PhasedArgs a{};
    a.k = (const __nv_bfloat16*)f.k;
    a.q = (const __nv_bfloat16*)f.q;
    a.v = (const __nv_bfloat16*)f.v;
    a.alpha = f.alpha;
    a.eta = f.eta;
    a.theta = f.theta;
    a.W1 = f.W1;
    a.W2 = f.W2;
    a.S1 = f.S1;
    a.S2 = f.S2;
    a.y = (__nv_bfloat16*)f.y;
    a.attn = (const __nv_bfloat16*)f.attn;
    a.ws = reinterpret_cast<uint8_t*>(f.ws);
    a.ws_stride = f.ws_per_unit * sizeof(float);
    a.T = f.T;
    a.gate_ld = f.gate_ld;
    a.chunk = f.chunk;
    a.units = (int)f.units;
    a.chunk_gates = f.chunk_gates ? 1 : 0;
    a.status = f.status;
    a.sync = sync;
    e = cudaMemsetAsync(sync, 0, 2 * sizeof(unsigned), st);
    if (e != cudaSuccess) return e;
    void* params[] = {&a};
    return cudaLaunchCooperativeKernel((const void*)chunk_fwd_tc_phased, dim3((unsigned)sm_count[dev].load()),
                                       dim3(ph::kThreads), params, ph::kSmemBytes, st);
}

}  // namespace titans
