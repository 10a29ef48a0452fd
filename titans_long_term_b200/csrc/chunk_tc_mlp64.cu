// Tensor-core chunk kernel for the MLP memory M(x) = W2 silu(W1 x), d = 64, h = 256,
// chunk n <= 64, bf16 operands with fp32 accumulation, fp32 state.
//
// Method ("Titans: Learning to Memorize at Test Time", walk-through sec. 3.1-3.2):
// per chunk every token's gradient of ||M(k) - v||^2 is taken at the chunk-start
// weights, so the chunk's momentum / forgetting recurrence folds into
//   W <- A W + sigma S - sum_j c_j g_j,   S <- E S - sum_j d_j g_j
// with per-token c_j, d_j and per-chunk A, E, sigma from a division-free suffix scan
// of the gates. The sums of per-token outer products are weighted GEMMs, so the
// whole chunk is five dense contractions on tcgen05:
//   Z^T     [h x 2n] = W1 [K;Q]^T          keys and queries through layer 1
//   Y       [2n x d] = silu(Z) W2^T         keys' M(k) and queries' retrieval
//   (GW2)^T [h x n]  = W2^T G^T             backprop of G = 2 (M(k) - v) to the hidden units
//   dW1     [h x d]  = Delta^T diag(-c|-d) K,  Delta = (G W2) * silu'(Z_K)
//   dW2^T   [h x d]  = A_K^T diag(-c|-d) G
// The hidden unit sits on the TMEM lane, so each thread of the epilogue warps owns one
// hidden row j of every state matrix:
//   - W1[j, :] and W2[:, j] (fp32) live in that thread's registers (W1 at half scale, so
//     the Z GEMM yields h = z/2, the argument of tanh in silu(z) = h (1 + tanh h)),
//   - S1[j, :] (half scale) and S2[:, j] (fp32) live in TMEM and are the accumulators of
//     the d-weighted GEMMs,
//   - the bf16 copies of W1 and W2^T that feed the MMAs are rewritten in shared memory
//     once per chunk.
// Per chunk, on the epilogue warps: SiLU of Z (keys also silu'); the momentum pre-pass
// W <- A W + sigma S (reads S only) while the tensor core computes Y; G and y; Delta;
// W += dW_c and the bf16 rows. The decay S <- E S is done by the four producer warps, one
// TMEM lane quadrant each; the d-weighted GEMMs (S accumulation) are issued after the
// weight GEMMs, off the weight-update path.
// Warp roles (12 warps, one CTA per SM, persistent over the chunk loop of one unit):
//   - warps 0-3 own hidden rows 0..127 ("tile 0"), warps 4-7 rows 128..255 ("tile 1");
//   - warps 8 and 9 issue tile 0's and tile 1's forward, backprop and W1-side MMAs (one
//     elected lane each: a single thread issues a tcgen05.mma only every ~100 cycles,
//     so more issuers shorten each MMA phase); Y is split into the two tiles' partial sums
//     over their hidden units, so those issuers never need ordering; warp 8 also issues
//     the TMA loads (K, Q, V two chunks ahead);
//   - warp 11 issues both tiles' W2-side weight GEMMs (dW2^T_c, then S2^T accumulation);
//   - warp 10 prefetches the gates, runs the gate scan a chunk ahead and writes the scaled
//     key tiles. The producer warpgroup (warps 8-11) hands registers to the epilogue
//     warpgroups (setmaxnreg).
// Hand-offs go through mbarriers only; every wait is bounded.
#include <cuda_bf16.h>
#include <algorithm>
#include <atomic>
#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace titans {

namespace tc {
constexpr int kEpiWarps = 8;
constexpr int kThreads = 384;  // 3 warpgroups: tile 0, tile 1, producer (warp 8 works, 9..11 idle)
// Register split: launched at kRegsLaunch per thread, the producer warpgroup gives registers
// back and the two epilogue warpgroups take them: 128 * kRegsProducer + 256 * kRegsEpilogue
// must not exceed 384 * kRegsLaunch (the block's launch allocation).
constexpr int kRegsLaunch = 168, kRegsProducer = 88, kRegsEpilogue = 208;
static_assert(128 * kRegsProducer + 256 * kRegsEpilogue <= 384 * kRegsLaunch, "register split");
constexpr int kD = 64, kH = 256, kN = 64;
// SiLU split between the special-function unit and the FMA pipe: of each 16-column block of the
// queries, the first kQueryFma columns take the FMA-pipe tanh (about 15 instructions instead of
// one MUFU op). Measured on the 128-unit, 4096-token workload, shares of 4, 6 and 8 columns take
// a launch from 0.409 ms to 0.419, 0.424 and 0.440 ms: the phase is not bound by the MUFU's
// throughput, so every evaluation stays on it (0 compiles to the MUFU-only loop).
constexpr int kQueryFma = 0;
// Shared-memory map (byte offsets from a 1024-aligned base). Every tile is
// [rows][64] bf16 with the 128-byte swizzle: 128 B per row, 1024-B atoms of 8 rows.
constexpr uint32_t W1 = 0;             // [256 h][64 d]      A of Z^T (K-major)
constexpr uint32_t W2T = W1 + 32768;   // [256 h][64 d]      A of (GW2)^T (K-major), B of Y (MN-major)
constexpr uint32_t KQ0 = W2T + 32768;  // [128 tok][64 d]    K rows 0..63, Q rows 64..127: B of Z^T
constexpr uint32_t KQ1 = KQ0 + 16384;
constexpr uint32_t V0 = KQ1 + 16384;   // [64 tok][64 d]
constexpr uint32_t V1 = V0 + 8192;
constexpr uint32_t AT0 = V1 + 8192;    // [256 h][64 tok]    silu(Z_K)^T: A of Y (MN-major), A of dW2^T
constexpr uint32_t AT1 = AT0 + 32768;  // [256 h][64 tok]    silu(Z_Q)^T for Y, then Delta^T (A of dW1)
constexpr uint32_t G = AT1 + 32768;    // [64 tok][64 d]     B of (GW2)^T (K-major)
constexpr uint32_t GC = G + 8192;      // -c_t G[t, :]       B of dW2^T (MN-major)
constexpr uint32_t GD = GC + 8192;     // -d_t G[t, :]
constexpr uint32_t KC = GD + 8192;     // -c_t K[t, :]       B of dW1 (MN-major)
constexpr uint32_t KD = KC + 8192;     // -d_t K[t, :]
constexpr uint32_t GATES = KD + 8192;  // staging for the scan: alpha, eta, theta [3][64] floats
constexpr uint32_t CC = GATES + 768;   // c_j  [2 parities][64]
constexpr uint32_t DD = CC + 512;      // d_j  [2][64]
constexpr uint32_t SCAL = DD + 512;    // A, E, sigma [2][4]
constexpr uint32_t BAR = SCAL + 32;    // mbarriers, 8 B each
enum Bar {
    B_TMA0, B_TMA1,      // K, Q, V tiles landed (buffer 0 / 1)
    B_Z0, B_Z1,          // Z^T of tile t done
    B_A0, B_A1,          // tile t wrote its silu rows (and silu' into TMEM)
    B_Y0, B_Y1,          // partial Y of tile t (sum over its hidden units) done
    B_G,                 // G tiles written, Y read (all epilogue threads)
    B_S0, B_S1,          // tile t's momentum pre-pass done
    B_GW0, B_GW1,        // (GW2)^T of tile t done
    B_D0, B_D1,          // tile t wrote Delta^T rows
    B_DW0, B_DW1,        // dW1_c of tile t done
    B_DX0, B_DX1,        // dW2^T_c of tile t done
    B_W0, B_W1,          // tile t rewrote its bf16 weight rows (and read dW1_c, dW2^T_c)
    B_SC0, B_SC1,        // gate scan of a chunk with parity 0 / 1 published
    B_KC,                // scaled key tiles of the chunk written
    B_RS,                // the four producer warps scaled S <- E S for the chunk
    B_SA0, B_SA1,        // S1 and S2^T accumulations of tile t done (a commit from each issuer)
    kNumBars
};
constexpr uint32_t TPTR = BAR + 8 * kNumBars;  // TMEM base address
constexpr uint32_t FLAG = TPTR + 4;            // abort flag
constexpr uint32_t END = FLAG + 4;
constexpr size_t kSmemBytes = END + 1024;  // + alignment slack
// TMEM columns: [0, 256) working region, [256, 512) momentum S.
//   working, tile t (hidden rows 128t..128t+127) at column 128t:
//     +0..63   Z_K^T, then silu'(Z_K)^T, then dW1_c
//     +64..127 Z_Q^T, then the partial Y of tile t, then (GW2)^T, then dW2^T_c
//   S region, tile t at column 256 + 128t: +0..63 S1 rows, +64..127 S2^T rows.
constexpr uint32_t kTmemCols = 512;
}  // namespace tc

static_assert(tc::kSmemBytes <= 232448, "shared memory budget");

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// 16-byte global -> shared copy (cached in L2 only) and the wait for all of a thread's copies.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit_wait() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ float ld_shared_f32(uint32_t a) {
    float x;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(x) : "r"(a) : "memory");
    return x;
}
__device__ __forceinline__ void st_shared_f32(uint32_t a, float x) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(x) : "memory");
}
// Named barrier of one epilogue warpgroup (tile t: barrier 1 + t, its 128 threads). The ids are
// immediates: with a register id ptxas reserves all sixteen barriers, and the chunk loop measured
// about 1% slower per chunk.
__device__ __forceinline__ void tile_bar(int tile) {
    if (tile == 0)
        asm volatile("bar.sync 1, 128;" ::: "memory");
    else
        asm volatile("bar.sync 2, 128;" ::: "memory");
}

// Writes 16 fp32 values as bf16 into columns [16 blk, 16 blk + 16) of row `row` of a
// swizzled [rows][64] tile (two 16-byte chunks).
__device__ __forceinline__ void store16_bf16(uint32_t tile, int row, int blk, const float* x) {
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
        const uint32_t a = tile + (uint32_t)row * 128u + ((uint32_t)((2 * blk + ch) ^ (row & 7)) << 4);
        st_shared_v4(a, pack_bf16x2(x[8 * ch + 0], x[8 * ch + 1]), pack_bf16x2(x[8 * ch + 2], x[8 * ch + 3]),
                     pack_bf16x2(x[8 * ch + 4], x[8 * ch + 5]), pack_bf16x2(x[8 * ch + 6], x[8 * ch + 7]));
    }
}

// Suffix scan of one chunk's gates (warp-wide, 2 tokens per lane, n <= 64, division-free):
//   P_j = prod_{l>j} (1 - alpha_l), Q_j = prod_{l>j} eta_l,
//   r_{n-1} = 1, r_j = P_j + eta_{j+1} r_{j+1}  (an affine suffix recurrence, scanned by
//   composing the maps r -> a r + b), c_j = theta_j r_j, d_j = theta_j Q_j,
//   A = (1 - alpha_0) P_0, E = eta_0 Q_0, sigma = eta_0 r_0.
// Tokens j >= n are padding: c_j = d_j = 0 and they leave every product unchanged.
__device__ __forceinline__ void gate_scan(int n, const float* sa, const float* se, const float* sth, float* cc,
                                          float* dd, float* scal, int lane) {
    const unsigned FULL = 0xffffffffu;
    const int j0 = 2 * lane, j1 = j0 + 1;
    const float om0 = j0 < n ? 1.f - sa[j0] : 1.f, om1 = j1 < n ? 1.f - sa[j1] : 1.f;
    const float et0 = j0 < n ? se[j0] : 1.f, et1 = j1 < n ? se[j1] : 1.f;
    float pp = om0 * om1, pq = et0 * et1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float a = __shfl_down_sync(FULL, pp, off), b = __shfl_down_sync(FULL, pq, off);
        if (lane + off < 32) {
            pp *= a;
            pq *= b;
        }
    }
    float exP = __shfl_down_sync(FULL, pp, 1), exQ = __shfl_down_sync(FULL, pq, 1);
    if (lane == 31) {
        exP = 1.f;
        exQ = 1.f;
    }
    const float P1 = exP, P0 = exP * om1, Q1 = exQ, Q0 = exQ * et1;
    const float b0 = j0 < n ? P0 : 0.f, b1 = j1 < n ? P1 : 0.f;
    const float a0 = j1 < n ? et1 : 0.f;
    const float eta_next = __shfl_down_sync(FULL, et0, 1);
    const float a1 = (j1 + 1 < n) ? eta_next : 0.f;
    float A = a0 * a1, Bv = b0 + a0 * b1;  // this lane's map applied to r_{j1+1}
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float A2 = __shfl_down_sync(FULL, A, off), B2 = __shfl_down_sync(FULL, Bv, off);
        if (lane + off < 32) {
            Bv = Bv + A * B2;
            A = A * A2;
        }
    }
    float Rnext = __shfl_down_sync(FULL, Bv, 1);
    if (lane == 31) Rnext = 0.f;
    const float r0 = Bv, r1 = b1 + a1 * Rnext;
    const float th0 = j0 < n ? sth[j0] : 0.f, th1 = j1 < n ? sth[j1] : 0.f;
    cc[j0] = th0 * r0;
    cc[j1] = th1 * r1;
    dd[j0] = th0 * Q0;
    dd[j1] = th1 * Q1;
    if (lane == 0) {
        scal[0] = om0 * P0;
        scal[1] = et0 * Q0;
        scal[2] = et0 * r0;
    }
}

// tanh via the hardware approximation (one MUFU op, relative error about 2^-11, below the
// bf16 rounding the activations get next).
__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// tanh|h| on the FMA and integer pipes only, so that part of the SiLU's evaluations leave the
// special-function unit, the bound of the SiLU phase, to run beside it. With e = exp(-2|h|) = 2^-y:
// 2^-y = 2^-n 2^-f (n = round(y) by the 1.5 * 2^23 rounding constant, f in [-1/2, 1/2], 2^-f a cubic,
// 2^-n subtracted from the exponent field), then tanh|h| = (1 - e) / (1 + e) as a quintic in
// e in [0, 1]. Both polynomials are Chebyshev interpolants generated by the fit script of this
// package (titans_long_term_b200/silu_fit.py); the absolute error is below 1.1e-4 (2^-13.2) for
// every fp32 h.
namespace tanh_fma {
constexpr float kP0 = 9.999245405e-01f, kP1 = -6.931367517e-01f, kP2 = 2.426394820e-01f, kP3 = -5.583828315e-02f;
constexpr float kQ0 = 9.998979568e-01f, kQ1 = -1.992551446e+00f, kQ2 = 1.906841516e+00f, kQ3 = -1.541145802e+00f, kQ4 = 8.358757496e-01f, kQ5 = -2.089689374e-01f;
constexpr float kLog2eX2 = 2.885390082f, kYMax = 64.f, kRound = 12582912.f;
}  // namespace tanh_fma
__device__ __forceinline__ float tanh_abs_fma(float h) {
    using namespace tanh_fma;
    const float y = fminf(fabsf(h) * kLog2eX2, kYMax);
    const float r = y + kRound;
    const float f = y - (r - kRound);
    const float p = fmaf(fmaf(fmaf(kP3, f, kP2), f, kP1), f, kP0);
    // 0 <= n <= 64 sits in the low bits of r; (bits(r) << 23) mod 2^32 = n << 23.
    const float e = __uint_as_float(__float_as_uint(p) - (__float_as_uint(r) << 23));
    return fmaf(fmaf(fmaf(fmaf(fmaf(kQ5, e, kQ4), e, kQ3), e, kQ2), e, kQ1), e, kQ0);
}
// silu(2h) = h (1 + tanh h) = h + |h| tanh|h| on that route.
__device__ __forceinline__ float silu_half_fma(float h) { return fmaf(fabsf(h), tanh_abs_fma(h), h); }

template <bool kCkpt>  // kCkpt: also write every chunk-start state to ckpt (the backward's first pass)
__global__ void __launch_bounds__(tc::kThreads, 1) chunk_fwd_tc_mlp64(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
    const __grid_constant__ CUtensorMap tmV, const float* __restrict__ alpha, const float* __restrict__ eta,
    const float* __restrict__ theta, float* __restrict__ W1g, float* __restrict__ W2g, float* __restrict__ S1g,
    float* __restrict__ S2g, __nv_bfloat16* __restrict__ yg, const __nv_bfloat16* __restrict__ attn, long T,
    long gate_ld, int chunk, int chunk_gates, unsigned* status, float* __restrict__ ckpt, long ckpt_stride) {
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + FLAG);
    float* s_cc = reinterpret_cast<float*>(sm + CC);
    float* s_dd = reinterpret_cast<float*>(sm + DD);
    float* s_scal = reinterpret_cast<float*>(sm + SCAL);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long u = blockIdx.x;
    const int nchunks = (int)((T + chunk - 1) / chunk);

    if (tid == 0) {
        for (int b = 0; b < kNumBars; ++b) {
            uint32_t cnt = 1;
            if (b == B_A0 || b == B_A1 || b == B_S0 || b == B_S1 || b == B_D0 || b == B_D1 || b == B_W0 ||
                b == B_W1)
                cnt = 128;
            else if (b == B_G)
                cnt = 256;
            else if (b == B_SC0 || b == B_SC1 || b == B_KC)
                cnt = 32;
            else if (b == B_RS)
                cnt = 4;
            else if (b == B_SA0 || b == B_SA1)
                cnt = 2;
            mbar_init(&bars[b], cnt);
        }
        fence_mbar_init();
        *abort_flag = 0;
    }
    if (warp == 0) {
        tmem_alloc(reinterpret_cast<uint32_t*>(sm + TPTR), kTmemCols);
        tmem_relinquish();
    }
    // Token tiles start at zero: rows beyond the chunk length are never written by TMA.
    for (uint32_t o = tid * 16; o < 49152; o += kThreads * 16) st_shared_v4(sb + KQ0 + o, 0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + TPTR);

#define DBG(cond) TITANS_DBG(cond, status, abort_flag)
    // TMEM column of an address relative to the allocation, and the byte span of shared memory in use.
    auto tcol_ok = [&](uint32_t taddr) { return ((taddr & 0xFFFFu) - (tmem & 0xFFFFu)) + 16u <= kTmemCols && (taddr >> 16) <= 96u; };
    auto smem_ok = [&](uint32_t addr) { return addr >= sb && addr + 16u <= sb + END; };
    // Bounded wait; on a timeout records the fault, raises the abort flag and returns false.
    auto wait = [&](int b, uint32_t parity) -> bool {
        if (mbar_wait(&bars[b], parity)) return true;
        atomicOr(status, b <= B_TMA1 ? kStatusTimeoutTma : kStatusTimeoutMma);
        *abort_flag = 1;
        return false;
    };

    if (warp >= kEpiWarps) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
    }
    // Momentum decay of chunk c, S <- E S, run by each producer warp on the S columns of both
    // tiles in its TMEM lane quadrant, after both tiles' pre-passes have read S (B_S); this
    // chunk's S accumulation waits for all four (B_RS). Returns false on a timeout.
    auto rescale_s = [&](int c) -> bool {
        const int p = c & 1;
        if (!wait(B_SC0 + p, (uint32_t)(c >> 1) & 1u)) return false;
        if (!wait(B_S0, (uint32_t)c & 1u) || !wait(B_S1, (uint32_t)c & 1u)) return false;
        tc_fence_after();
        const float En = s_scal[4 * p + 1];
        const uint32_t tq = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + 256;
        // 32 columns per TMEM round trip (16 measured 1% slower per launch; 64 spill at 88 registers)
#pragma unroll 1
        for (int col = 0; col < 256; col += 32) {
            uint32_t r[32];
            tmem_ld32(tq + col, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(En * __uint_as_float(r[i]));
            tmem_st32(tq + col, r);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_RS]);
        return true;
    };
    if (warp == kEpiWarps + 2) {
        // =========================== scan warp: gates, gate scans, scaled key tiles
        float ga[2], ge[2], gt[2];  // gates of one chunk, lane l holds tokens l and l + 32
        auto load_gates = [&](int c) {
            const long t0 = (long)c * chunk;
            const long n = c < nchunks ? min((long)chunk, T - t0) : 0;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int j = lane + 32 * i;
                const bool ok = j < n;
                const long g = u * gate_ld + (chunk_gates ? (long)c : t0 + j);  // chunk-shared or per-token
                const bool in = ok && DBG(g >= u * gate_ld && g < (u + 1) * gate_ld);
                ga[i] = in ? __ldg(alpha + g) : 0.f;
                ge[i] = in ? __ldg(eta + g) : 1.f;
                gt[i] = in ? __ldg(theta + g) : 0.f;
            }
        };
        float* sg = reinterpret_cast<float*>(sm + GATES);
        auto scan = [&](int c) {  // gates of chunk c are in registers
            const long t0 = (long)c * chunk;
            const int n = (int)min((long)chunk, T - t0);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                sg[lane + 32 * i] = ga[i];
                sg[64 + lane + 32 * i] = ge[i];
                sg[128 + lane + 32 * i] = gt[i];
            }
            __syncwarp();
            const int p = c & 1;
            gate_scan(n, sg, sg + 64, sg + 128, s_cc + 64 * p, s_dd + 64 * p, s_scal + 4 * p, lane);
            __syncwarp();
            mbar_arrive(&bars[B_SC0 + p]);
        };
        load_gates(0);
        scan(0);
        load_gates(1);
        for (int c = 0; c < nchunks; ++c) {
            const int p = c & 1;
            const uint32_t KQb = (c & 1) ? KQ1 : KQ0;
            if (!wait(B_TMA0 + (c & 1), (uint32_t)(c >> 1) & 1u)) break;
            // The previous chunk's S1 accumulations of both tiles (the last readers of the scaled
            // key tiles; every reader of the other scan buffer finished before them) have completed.
            if (c > 0 && (!wait(B_SA0, (uint32_t)(c - 1) & 1u) || !wait(B_SA1, (uint32_t)(c - 1) & 1u))) break;
            {
                const float* cc = s_cc + 64 * p;
                const float* dd = s_dd + 64 * p;
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    const uint32_t off = (uint32_t)(lane + 32 * i) * 16u;
                    const int row = (lane + 32 * i) >> 3;
                    if (!DBG(off + 16u <= 8192u)) continue;
                    const uint4 kv = ld_shared_v4(sb + KQb + off);
                    const float cr = -0.5f * cc[row], dr = -0.5f * dd[row];  // W1, S1 are kept halved
                    const uint32_t in[4] = {kv.x, kv.y, kv.z, kv.w};
                    uint32_t oc[4], od[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = unpack_bf16x2(in[e]);
                        oc[e] = pack_bf16x2(cr * f.x, cr * f.y);
                        od[e] = pack_bf16x2(dr * f.x, dr * f.y);
                    }
                    st_shared_v4(sb + KC + off, oc[0], oc[1], oc[2], oc[3]);
                    st_shared_v4(sb + KD + off, od[0], od[1], od[2], od[3]);
                }
                fence_proxy_async_smem();
                mbar_arrive(&bars[B_KC]);
            }
            if (!rescale_s(c)) break;
            if (c + 1 < nchunks) {
                scan(c + 1);
                load_gates(c + 2);
            }
        }
    } else if (warp == kEpiWarps + 3) {
        // =========================== W2-side issuer: S2^T += A_K^T diag(-d) G, dW2^T_c = A_K^T diag(-c) G
        const uint32_t idW = idesc_bf16_f32(128, 64, 0, 1);
        const uint64_t dK = sdesc_sw128(sb, 16, 1024);
        const uint64_t dMN8 = sdesc_sw128(sb, 8192, 1024);
#define DSC(base, off) ((base) + (uint64_t)((off) >> 4))
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t ph = (uint32_t)c & 1u;
            bool ok = rescale_s(c);
            ok = ok && wait(B_G, ph);  // G and its scaled copies written
            // dW2^T_c of tile t into columns 128t+64 once the Delta epilogue has read (GW2)^T there.
            for (int t = 0; t < 2 && ok; ++t) {
                ok = wait(B_D0 + t, ph);
                if (ok && lane == 0) {
                    tc_fence_after();
#pragma unroll 1
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(tmem + t * 128 + 64, DSC(dK, AT0 + t * 16384 + ks * 32),
                                  DSC(dMN8, GC + ks * 2048), idW, ks > 0);
                    umma_commit(&bars[B_DX0 + t]);
                }
            }
            // S2^T accumulation of tile t (S already scaled by E, B_RS): off the weight-update
            // path, it runs while the epilogue rewrites the weights; the next chunk's SiLU
            // (which overwrites A_K) waits for B_SA.
            ok = ok && wait(B_RS, ph);
            for (int t = 0; t < 2 && ok; ++t) {
                if (lane == 0) {
                    tc_fence_after();
#pragma unroll 1
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(tmem + 256 + t * 128 + 64, DSC(dK, AT0 + t * 16384 + ks * 32),
                                  DSC(dMN8, GD + ks * 2048), idW, 1);
                    umma_commit(&bars[B_SA0 + t]);
                }
            }
            if (!ok) break;
            __syncwarp();
        }
#undef DSC
    } else if (warp >= kEpiWarps) {
        // =========================== issuer warps: warp 8 + t issues tile t's MMAs (warp 8 also TMA)
        const int t = warp - kEpiWarps;
        const uint32_t idZ = idesc_bf16_f32(128, 128, 0, 0);
        const uint32_t idY = idesc_bf16_f32(128, 64, 1, 1);
        const uint32_t idG = idesc_bf16_f32(128, 64, 0, 0);
        const uint32_t idW = idesc_bf16_f32(128, 64, 0, 1);
        const uint32_t tx_bytes = 3u * (uint32_t)chunk * 128u;
        // Descriptor bases at offset 0 of shared memory; a tile at byte offset X is base + X / 16
        // (the start-address field is the low 14 bits and every address stays below 256 KB).
        const uint64_t dK = sdesc_sw128(sb, 16, 1024);            // K-major, 8-row groups 1024 B apart
        const uint64_t dMN32 = sdesc_sw128(sb, AT1 - AT0, 1024);  // MN-major, 64-element blocks 32 KB apart
        const uint64_t dMN8 = sdesc_sw128(sb, 8192, 1024);        // MN-major, single 64-element block
#define DSC(base, off) ((base) + (uint64_t)((off) >> 4))
        uint32_t tma_issued = 0, tma_waited = 0;  // counts per buffer packed: bits [0,16) buf 0, [16,32) buf 1
        auto issue_tma = [&](int c) {
            const int b = c & 1;
            const uint32_t kq = b ? KQ1 : KQ0, vv = b ? V1 : V0;
            // coordinates: x = 0 (16-byte aligned), a token row inside the stream, this unit
            if (!DBG((long)c * chunk < T && u < (long)gridDim.x)) return;
            mbar_arrive_expect_tx(&bars[B_TMA0 + b], tx_bytes);
            tma_load_3d(sm + kq, &tmK, &bars[B_TMA0 + b], 0, c * chunk, (int)u);
            tma_load_3d(sm + kq + 8192, &tmQ, &bars[B_TMA0 + b], 0, c * chunk, (int)u);
            tma_load_3d(sm + vv, &tmV, &bars[B_TMA0 + b], 0, c * chunk, (int)u);
            tma_issued += b ? 0x10000u : 1u;
        };
        if (t == 0 && lane == 0) {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmV);
            issue_tma(0);
            if (nchunks > 1) issue_tma(1);
        }
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const uint32_t ph = (uint32_t)c & 1u;
            const uint32_t KQb = b ? KQ1 : KQ0;
            bool ok = wait(B_TMA0 + b, (uint32_t)(c >> 1) & 1u);
            if (ok) tma_waited += b ? 0x10000u : 1u;
            // Z^T of tile t once tile t has rewritten its weight rows (after chunk c-1).
            if (ok) ok = wait(B_W0 + t, ph);
            if (ok && lane == 0) {
                tc_fence_after();
#pragma unroll 1
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(tmem + t * 128, DSC(dK, W1 + t * 16384 + ks * 32), DSC(dK, KQb + ks * 32), idZ, ks > 0);
                umma_commit(&bars[B_Z0 + t]);
            }
            if (!ok || *abort_flag) break;
            // Partial Y of tile t: its 128 hidden units are K-steps 8t .. 8t+7 of A W2^T.
            ok = wait(B_A0 + t, ph);
            if (ok && lane == 0) {
                tc_fence_after();
#pragma unroll 1
                for (int j = 0; j < 8; ++j)
                    umma_bf16(tmem + t * 128 + 64, DSC(dMN32, AT0 + (8 * t + j) * 2048),
                              DSC(dMN8, W2T + (8 * t + j) * 2048), idY, j > 0);
                umma_commit(&bars[B_Y0 + t]);
            }
            if (!ok) break;
            __syncwarp();
            if (!rescale_s(c)) break;
            ok = wait(B_G, ph);  // G tiles written, both partial Y read
            if (!ok) break;
            // (GW2)^T = W2^T G^T.
            if (lane == 0) {
                tc_fence_after();
#pragma unroll 1
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(tmem + t * 128 + 64, DSC(dK, W2T + t * 16384 + ks * 32), DSC(dK, G + ks * 32), idG,
                              ks > 0);
                umma_commit(&bars[B_GW0 + t]);
            }
            // Scaled key tiles written: with the G tiles written before, every reader of this
            // chunk's K, Q, V buffer is done -> chunk c + 2.
            ok = wait(B_KC, ph);
            if (ok && t == 0 && lane == 0 && c + 2 < nchunks) issue_tma(c + 2);
            // dW1_c -> cols 128t and S1 += Delta^T diag(-d) K once S is pre-scaled and Delta^T written.
            if (ok) ok = wait(B_RS, ph) && wait(B_D0 + t, ph);
            if (ok && lane == 0) {
                tc_fence_after();
#pragma unroll 1
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(tmem + t * 128, DSC(dK, AT1 + t * 16384 + ks * 32), DSC(dMN8, KC + ks * 2048), idW,
                              ks > 0);
                umma_commit(&bars[B_DW0 + t]);
                // S1 accumulation after the weight GEMM: the weight update waits for dW1_c only.
#pragma unroll 1
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(tmem + 256 + t * 128, DSC(dK, AT1 + t * 16384 + ks * 32), DSC(dMN8, KD + ks * 2048),
                              idW, 1);
                umma_commit(&bars[B_SA0 + t]);
            }
            if (!ok) break;
            __syncwarp();
        }
#undef DSC
        __syncwarp();
        // Drain: after an abort, copies may still be in flight into shared memory.
        if (t == 0 && lane == 0) {
            for (int b = 0; b < 2; ++b) {
                uint32_t iss = (tma_issued >> (16 * b)) & 0xFFFFu, don = (tma_waited >> (16 * b)) & 0xFFFFu;
                while (don < iss) {
                    if (!mbar_wait(&bars[B_TMA0 + b], don & 1u)) break;
                    ++don;
                }
            }
        }
    } else {
        // =========================== epilogue warps: one hidden row per thread
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpilogue));
        const int quad = warp & 3, tile = warp >> 2;
        const int hrow = tile * 128 + quad * 32 + lane;
        const uint32_t lane_off = uint32_t(quad * 32) << 16;
        const uint32_t t_work = tmem + lane_off + tile * 128;     // this tile's working columns
        const uint32_t t_s = tmem + lane_off + 256 + tile * 128;  // S1 at +0, S2^T at +64
        float w1[64], w2[64];
        // The unit's state moves between global memory and the threads' rows through shared memory
        // that the tile does not use at entry or exit, so that every global access is coalesced:
        //   region A (this tile's AT0 and AT1 rows, 32 KB): a row-major [128][64] fp32 block of W1 or S1,
        //     row r at r * 256 B with its 16-byte pieces XORed by r & 15 (conflict-free row reads);
        //   region B (this tile's bf16 W1 and W2^T rows, 32 KB): the tile's 128 columns of W2 or S2,
        //     [64][128] fp32 (a thread's column reads are conflict-free as they stand).
        const int it = hrow - 128 * tile;  // the thread's row within the tile
        auto a_addr = [&](int r, int c) -> uint32_t {
            return sb + (r < 64 ? AT0 : AT1) + (uint32_t)tile * 16384u + (uint32_t)(r & 63) * 256u +
                   ((uint32_t)(c ^ (r & 15)) << 4);
        };
        auto b_addr = [&](int d, int col) -> uint32_t {
            return sb + (d < 32 ? W1 : W2T) + (uint32_t)tile * 16384u + (uint32_t)(d & 31) * 512u + (uint32_t)col * 4u;
        };
        // global -> regions A, B: the tile's rows of a [256][64] matrix (32 KB, contiguous) and the
        // tile's columns of a [64][256] matrix (64 rows of 512 B), 16-byte copies all in flight
        auto stage_in_state = [&](const float* rows, const float* cols) {
            const float* ga = rows + (u * kH + 128 * tile) * kD;
            const float* gb = cols + u * kD * kH + 128 * tile;
            for (int q = it; q < 2048; q += 128) {
                cp_async_16(a_addr(q >> 4, q & 15), ga + 4 * q);
                cp_async_16(b_addr(q >> 5, 4 * (q & 31)), gb + (q >> 5) * kH + 4 * (q & 31));
            }
            cp_async_commit_wait();
            tile_bar(tile);
        };
        // regions A, B -> global, the same layouts, coalesced 16-byte stores
        auto stage_out_state = [&](float* rows, float* cols) {
            tile_bar(tile);
            float* ga = rows + (u * kH + 128 * tile) * kD;
            float* gb = cols + u * kD * kH + 128 * tile;
            for (int q = it; q < 2048; q += 128) {
                const uint4 x = ld_shared_v4(a_addr(q >> 4, q & 15));
                *reinterpret_cast<uint4*>(ga + 4 * q) = x;
                const uint4 y2 = ld_shared_v4(b_addr(q >> 5, 4 * (q & 31)));
                *reinterpret_cast<uint4*>(gb + (q >> 5) * kH + 4 * (q & 31)) = y2;
            }
            tile_bar(tile);
        };
        {
            // S first, straight into TMEM, so that nothing else is live while it passes through
            stage_in_state(S1g, S2g);
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
                uint32_t r[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 x = ld_shared_v4(a_addr(it, 4 * blk + j));
                    r[4 * j] = __float_as_uint(0.5f * __uint_as_float(x.x));
                    r[4 * j + 1] = __float_as_uint(0.5f * __uint_as_float(x.y));
                    r[4 * j + 2] = __float_as_uint(0.5f * __uint_as_float(x.z));
                    r[4 * j + 3] = __float_as_uint(0.5f * __uint_as_float(x.w));
                }
                tmem_st16(t_s + 16 * blk, r);
#pragma unroll
                for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(ld_shared_f32(b_addr(16 * blk + i, it)));
                tmem_st16(t_s + 64 + 16 * blk, r);
            }
            tile_bar(tile);  // every row read before the regions take W
            stage_in_state(W1g, W2g);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint4 x = ld_shared_v4(a_addr(it, i));
                w1[4 * i] = 0.5f * __uint_as_float(x.x);
                w1[4 * i + 1] = 0.5f * __uint_as_float(x.y);
                w1[4 * i + 2] = 0.5f * __uint_as_float(x.z);
                w1[4 * i + 3] = 0.5f * __uint_as_float(x.w);
            }
#pragma unroll
            for (int i = 0; i < 64; ++i) w2[i] = ld_shared_f32(b_addr(i, it));
            tile_bar(tile);  // region B is the bf16 W1 and W2^T rows written next
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
                store16_bf16(sb + W1, hrow, blk, w1 + 16 * blk);
                store16_bf16(sb + W2T, hrow, blk, w2 + 16 * blk);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_W0 + tile]);  // completion 0: the weights of "chunk -1"
        }

        for (int c = 0; c < nchunks; ++c) {
            const int p = c & 1;
            const uint32_t ph = (uint32_t)c & 1u;
            const long t0 = (long)c * chunk;
            const int n = (int)min((long)chunk, T - t0);

            // (1) A = silu(Z): keys -> AT0 (and silu'(Z_K) into TMEM), queries -> AT1
            if (!wait(B_Z0 + tile, ph)) break;
            // The previous chunk's S accumulations read this tile's A_K and Delta^T rows.
            if (c > 0 && !wait(B_SA0 + tile, (uint32_t)(c - 1) & 1u)) break;
            tc_fence_after();
#pragma unroll 1
            for (int blk = 0; blk < 4; ++blk) {  // keys and queries, 16-column blocks
                uint32_t rk[16], rq[16];
                if (!DBG(tcol_ok(t_work + 16 * blk) && tcol_ok(t_work + 64 + 16 * blk) &&
                         smem_ok(sb + AT1 + (uint32_t)hrow * 128u + 112u)))
                    break;
                tmem_ld16(t_work + 16 * blk, rk);
                tmem_ld16(t_work + 64 + 16 * blk, rq);
                tmem_wait_ld();
                uint32_t pk[8], pq[8];
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    // silu(z) = h (1 + tanh h), silu'(z) = (1 + tanh h + h (1 - tanh^2 h)) / 2, h = z / 2
                    const float h0 = __uint_as_float(rk[i]), h1 = __uint_as_float(rk[i + 1]);
                    const float t0_ = tanh_approx(h0), t1_ = tanh_approx(h1);
                    const float a0 = fmaf(h0, t0_, h0), a1 = fmaf(h1, t1_, h1);  // silu
                    const float s0 = fmaf(0.5f, t0_, 0.5f), s1 = fmaf(0.5f, t1_, 0.5f);  // sigmoid
                    pk[i / 2] = pack_bf16x2(a0, a1);
                    rk[i] = __float_as_uint(fmaf(-a0, s0, a0 + s0));  // silu' = sigma + silu (1 - sigma)
                    rk[i + 1] = __float_as_uint(fmaf(-a1, s1, a1 + s1));
                    // Queries: the first kQueryFma columns of a block take the FMA-pipe tanh.
                    const float g0 = __uint_as_float(rq[i]), g1 = __uint_as_float(rq[i + 1]);
                    const float q0 = i < kQueryFma ? silu_half_fma(g0) : fmaf(g0, tanh_approx(g0), g0);
                    const float q1 = i + 1 < kQueryFma ? silu_half_fma(g1) : fmaf(g1, tanh_approx(g1), g1);
                    pq[i / 2] = pack_bf16x2(q0, q1);
                }
                tmem_st16(t_work + 16 * blk, rk);
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    const uint32_t sw = (uint32_t)((2 * blk + ch) ^ (hrow & 7)) << 4;
                    st_shared_v4(sb + AT0 + (uint32_t)hrow * 128u + sw, pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2],
                                 pk[4 * ch + 3]);
                    st_shared_v4(sb + AT1 + (uint32_t)hrow * 128u + sw, pq[4 * ch], pq[4 * ch + 1], pq[4 * ch + 2],
                                 pq[4 * ch + 3]);
                }
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_A0 + tile]);

            // (2) momentum pre-pass while the tensor core runs Y: W <- A W + sigma S (reads S only;
            //     the producer warps then scale S <- E S, and the d-GEMMs add -sum d_j g_j)
            if (!wait(B_SC0 + p, (uint32_t)(c >> 1) & 1u)) break;
            {
                const float An = s_scal[4 * p], sig = s_scal[4 * p + 2];
                // Optional checkpoint of the chunk-start state (W in registers, S in TMEM), for the
                // backward's first pass: W1, S1 rows and W2, S2 columns of this thread's hidden row.
                float* ck = kCkpt ? ckpt + u * ckpt_stride + (long)c * 4 * kH * kD : nullptr;
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    uint32_t r1[16], r2[16];
                    tmem_ld16(t_s + 16 * blk, r1);
                    tmem_ld16(t_s + 64 + 16 * blk, r2);
                    tmem_wait_ld();
                    if (kCkpt) {
                        float4* c1 = reinterpret_cast<float4*>(ck + (size_t)hrow * kD + 16 * blk);
                        float4* s1 = reinterpret_cast<float4*>(ck + 2 * kH * kD + (size_t)hrow * kD + 16 * blk);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            c1[i] = make_float4(2.f * w1[16 * blk + 4 * i], 2.f * w1[16 * blk + 4 * i + 1],
                                                2.f * w1[16 * blk + 4 * i + 2], 2.f * w1[16 * blk + 4 * i + 3]);
                            s1[i] = make_float4(2.f * __uint_as_float(r1[4 * i]), 2.f * __uint_as_float(r1[4 * i + 1]),
                                                2.f * __uint_as_float(r1[4 * i + 2]), 2.f * __uint_as_float(r1[4 * i + 3]));
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            ck[kH * kD + (size_t)(16 * blk + i) * kH + hrow] = w2[16 * blk + i];
                            ck[3 * kH * kD + (size_t)(16 * blk + i) * kH + hrow] = __uint_as_float(r2[i]);
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        w1[16 * blk + i] = fmaf(An, w1[16 * blk + i], sig * __uint_as_float(r1[i]));
                        w2[16 * blk + i] = fmaf(An, w2[16 * blk + i], sig * __uint_as_float(r2[i]));
                    }
                }
                tc_fence_before();
                mbar_arrive(&bars[B_S0 + tile]);
            }

            // (3) G = 2 (M(k) - v) and its scaled copies (keys), y (queries). Token row = TMEM
            //     lane (quadrant quad), this warp's 32 of the 64 columns: [32 tile, 32 tile + 32).
            if (!wait(B_TMA0 + (c & 1), (uint32_t)(c >> 1) & 1u)) break;  // the V tile, read below
            if (!wait(B_Y0, ph) || !wait(B_Y1, ph)) break;
            tc_fence_after();
            {
                const int row = quad * 32 + lane;
                if (row < kN) {  // key row: G and its c- and d-scaled copies (bf16 tiles)
                    const uint32_t Vb = (c & 1) ? V1 : V0;
                    const float cr = -s_cc[64 * p + row], dr = -s_dd[64 * p + row];
#pragma unroll 1
                    for (int hb = 0; hb < 2; ++hb) {
                        const int col0 = 32 * tile + 16 * hb;
                        uint32_t r[16], r2[16];
                        tmem_ld16(tmem + lane_off + 64 + col0, r);         // tile 0's partial Y
                        tmem_ld16(tmem + lane_off + 128 + 64 + col0, r2);  // tile 1's partial Y
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            r[i] = __float_as_uint(__uint_as_float(r[i]) + __uint_as_float(r2[i]));
#pragma unroll
                        for (int ch = 0; ch < 2; ++ch) {
                            const uint32_t off = sw128_off((uint32_t)row, (uint32_t)(col0 + 8 * ch));
                            if (!DBG(off + 16u <= 8192u)) continue;
                            const uint4 vv = ld_shared_v4(sb + Vb + off);
                            const uint32_t vin[4] = {vv.x, vv.y, vv.z, vv.w};
                            uint32_t og[4], oc[4], od[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 vf = unpack_bf16x2(vin[e]);
                                const float g0 = 2.f * (__uint_as_float(r[8 * ch + 2 * e]) - vf.x);
                                const float g1 = 2.f * (__uint_as_float(r[8 * ch + 2 * e + 1]) - vf.y);
                                og[e] = pack_bf16x2(g0, g1);
                                oc[e] = pack_bf16x2(cr * g0, cr * g1);
                                od[e] = pack_bf16x2(dr * g0, dr * g1);
                            }
                            st_shared_v4(sb + G + off, og[0], og[1], og[2], og[3]);
                            st_shared_v4(sb + GC + off, oc[0], oc[1], oc[2], oc[3]);
                            st_shared_v4(sb + GD + off, od[0], od[1], od[2], od[3]);
                        }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(&bars[B_G]);
                } else {  // query row: y, stored after the arrival (the TMEM reads are what GW waits for)
                    float yv[32];
#pragma unroll
                    for (int hb = 0; hb < 2; ++hb) {
                        const int col0 = 32 * tile + 16 * hb;
                        uint32_t r[16], r2[16];
                        tmem_ld16(tmem + lane_off + 64 + col0, r);
                        tmem_ld16(tmem + lane_off + 128 + 64 + col0, r2);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) yv[16 * hb + i] = __uint_as_float(r[i]) + __uint_as_float(r2[i]);
                    }
                    tc_fence_before();
                    mbar_arrive(&bars[B_G]);
                    if (row - kN < n && DBG(t0 + (row - kN) < T)) {
                        const long off = (u * T + t0 + (row - kN)) * kD + 32 * tile;
                        uint4* dst = reinterpret_cast<uint4*>(yg + off);
                        if (attn == nullptr) {
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4)
                                dst[q4] = make_uint4(pack_bf16x2(yv[8 * q4], yv[8 * q4 + 1]),
                                                     pack_bf16x2(yv[8 * q4 + 2], yv[8 * q4 + 3]),
                                                     pack_bf16x2(yv[8 * q4 + 4], yv[8 * q4 + 5]),
                                                     pack_bf16x2(yv[8 * q4 + 6], yv[8 * q4 + 7]));
                        } else {
                            // The memory-as-a-gate output attn * sigmoid(y), sigmoid(y) = (1 + tanh(y / 2)) / 2
                            // ("Titans", walk-through sec. 4.2 "Gated Memory").
                            const uint4* arow = reinterpret_cast<const uint4*>(attn + off);
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4) {
                                const uint4 av = __ldg(arow + q4);
                                const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
                                uint32_t ow[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float2 a2 = unpack_bf16x2(aw[e]);
                                    const float y0 = yv[8 * q4 + 2 * e], y1 = yv[8 * q4 + 2 * e + 1];
                                    ow[e] = pack_bf16x2(a2.x * fmaf(0.5f, tanh_approx(0.5f * y0), 0.5f),
                                                        a2.y * fmaf(0.5f, tanh_approx(0.5f * y1), 0.5f));
                                }
                                dst[q4] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                            }
                        }
                    }
                }
            }

            // (4) Delta^T = (GW2)^T * silu'(Z_K)^T -> AT1 rows (the queries' tile was consumed by Y)
            if (!wait(B_GW0 + tile, ph)) break;
            tc_fence_after();
#pragma unroll 1
            for (int blk = 0; blk < 4; ++blk) {
                uint32_t g[16], sp[16];
                tmem_ld16(t_work + 64 + 16 * blk, g);
                tmem_ld16(t_work + 16 * blk, sp);
                tmem_wait_ld();
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = __uint_as_float(g[i]) * __uint_as_float(sp[i]);
                store16_bf16(sb + AT1, hrow, blk, x);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_D0 + tile]);

            // (5) W <- (A W + sigma S) - sum_j c_j g_j; rewrite the bf16 operand rows
            if (!wait(B_DW0 + tile, ph) || !wait(B_DX0 + tile, ph)) break;
            tc_fence_after();
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
                uint32_t r1[16], r2[16];
                tmem_ld16(t_work + 16 * blk, r1);
                tmem_ld16(t_work + 64 + 16 * blk, r2);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    w1[16 * blk + i] += __uint_as_float(r1[i]);
                    w2[16 * blk + i] += __uint_as_float(r2[i]);
                }
                store16_bf16(sb + W1, hrow, blk, w1 + 16 * blk);
            }
            // The next chunk's Z^T needs only the W1 rows; every TMEM read of dW1, dW2^T is done.
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_W0 + tile]);
            // W2^T rows after the arrival: their readers, Y and (GW2)^T, wait for this thread's later
            // arrivals (the SiLU's and G's), which follow these stores and a proxy fence.
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) store16_bf16(sb + W2T, hrow, blk, w2 + 16 * blk);
        }

        // Final state of this tile, once the last chunk's S accumulations (the last readers of the
        // tile's AT0 and AT1 rows) have completed; its bf16 weight rows are no longer read either.
        if (nchunks > 0 && !*abort_flag) wait(B_SA0 + tile, (uint32_t)(nchunks - 1) & 1u);
        // Region B is this tile's bf16 weight rows, which every thread of the tile rewrote in the
        // last chunk's weight update; the wait above does not order those stores, so all of the
        // tile's threads finish them before any staging write.
        tile_bar(tile);
        {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                st_shared_v4(a_addr(it, i), __float_as_uint(2.f * w1[4 * i]), __float_as_uint(2.f * w1[4 * i + 1]),
                             __float_as_uint(2.f * w1[4 * i + 2]), __float_as_uint(2.f * w1[4 * i + 3]));
#pragma unroll
            for (int i = 0; i < 64; ++i) st_shared_f32(b_addr(i, it), w2[i]);
            stage_out_state(W1g, W2g);
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
                uint32_t r[16];
                tmem_ld16(t_s + 16 * blk, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    st_shared_v4(a_addr(it, 4 * blk + j), __float_as_uint(2.f * __uint_as_float(r[4 * j])),
                                 __float_as_uint(2.f * __uint_as_float(r[4 * j + 1])),
                                 __float_as_uint(2.f * __uint_as_float(r[4 * j + 2])),
                                 __float_as_uint(2.f * __uint_as_float(r[4 * j + 3])));
                tmem_ld16(t_s + 64 + 16 * blk, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) st_shared_f32(b_addr(16 * blk + i, it), __uint_as_float(r[i]));
            }
            stage_out_state(S1g, S2g);
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

// Both SiLU routes of the chunk kernel, silu(2h) = h (1 + tanh h), on n arguments h.
__global__ void silu_routes_kernel(const float* __restrict__ h, float* __restrict__ s_fma,
                                   float* __restrict__ s_mufu, long n) {
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const float x = h[i];
        s_fma[i] = silu_half_fma(x);
        s_mufu[i] = fmaf(x, tanh_approx(x), x);
    }
}

cudaError_t launch_silu_routes(const float* h, float* s_fma, float* s_mufu, long n, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const long blocks = std::min<long>((n + 255) / 256, 148L * 8);
    silu_routes_kernel<<<(unsigned)blocks, 256, 0, st>>>(h, s_fma, s_mufu, n);
    return cudaGetLastError();
}

size_t chunk_tc_mlp64_smem_bytes() { return tc::kSmemBytes; }

cudaError_t launch_chunk_tc_mlp64(const ForwardArgs& a, const CUtensorMap& tk, const CUtensorMap& tq,
                                  const CUtensorMap& tv, cudaStream_t st) {
    // The shared-memory opt-in is per function and device: set it once per device.
    static std::atomic<unsigned long long> attr_set{0};
    int dev = 0;
    cudaError_t e0 = cudaGetDevice(&dev);
    if (e0 != cudaSuccess) return e0;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(attr_set.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(chunk_fwd_tc_mlp64<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)tc::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(chunk_fwd_tc_mlp64<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)tc::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(bit);
    }
    auto kernel = a.ckpt ? chunk_fwd_tc_mlp64<true> : chunk_fwd_tc_mlp64<false>;
    kernel<<<(unsigned)a.units, tc::kThreads, tc::kSmemBytes, st>>>(
        tk, tq, tv, a.alpha, a.eta, a.theta, a.W1, a.W2, a.S1, a.S2, (__nv_bfloat16*)a.y,
        (const __nv_bfloat16*)a.attn, a.T, a.gate_ld, a.chunk, (int)a.chunk_gates, a.status, a.ckpt,
        (long)a.ckpt_unit_stride);
    return cudaGetLastError();
}

}  // namespace titans
