// Tensor-core chunk kernel for the MLP memory M(x) = W2 silu(W1 x), d = 64, h = 256,
// chunk n <= 64, bf16 operands with fp32 accumulation, fp32 state.
//
// Method ("Titans: Learning to Memorize at Test Time", walk-through sec. 3.1-3.2):
// per chunk every token's gradient of ||M(k) - v||^2 is taken at the chunk-start
// weights, so the chunk's momentum / forgetting recurrence folds into
//   W <- A W + sigma S - sum_j c_j g_j,   S <- E S - sum_j d_j g_j
// with per-token c_j, d_j and per-chunk A, E, sigma from a division-free suffix scan
// of the gates. The sums of per-token outer products are two weighted GEMMs, so the
// whole chunk is five dense contractions on tcgen05:
//   Z^T   [h x 2n] = W1 [K;Q]^T          keys and queries through layer 1
//   Y     [2n x d] = silu(Z) W2^T         keys' M(k) and queries' retrieval
//   (GW2)^T [h x n] = W2^T G^T            backprop of G = 2 (M(k) - v) to the hidden units
//   dW1   [h x d] = Delta^T diag(-c|-d) K,  Delta = (G W2) * silu'(Z)
//   dW2^T [h x d] = A_K^T diag(-c|-d) G
// Everything is laid out with the hidden unit on the TMEM lane, so each thread owns
// one hidden row j of every state matrix:
//   - W1[j, :] and W2[:, j] (fp32) live in that thread's registers,
//   - S1[j, :] and S2[:, j] (fp32) live in TMEM and are the accumulators of the
//     d-weighted GEMMs (pre-scaled by E before the GEMM accumulates -sum d_j g_j),
//   - the bf16 copies of W1 and W2^T that feed the MMAs are rewritten in shared
//     memory once per chunk.
// One CTA (8 warps, 1 per SM) per (batch, head) unit, persistent over the chunk loop;
// K, Q, V tiles of chunk c+2 stream in by TMA while chunk c computes.
#include <cuda_bf16.h>
#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace titans {

namespace tc {
constexpr int kThreads = 256;
constexpr int kD = 64, kH = 256, kN = 64;
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
constexpr uint32_t ALPHA = KD + 8192;  // 64 floats each
constexpr uint32_t ETA = ALPHA + 256;
constexpr uint32_t THETA = ETA + 256;
constexpr uint32_t CC = THETA + 256;
constexpr uint32_t DD = CC + 256;
constexpr uint32_t SCAL = DD + 256;    // A, E, sigma
constexpr uint32_t BAR = SCAL + 16;    // tma[0], tma[1], mma: 3 x u64
constexpr uint32_t TPTR = BAR + 24;    // TMEM base address
constexpr uint32_t FLAG = TPTR + 4;    // abort flag
constexpr uint32_t END = FLAG + 4;
constexpr size_t kSmemBytes = END + 1024;  // + alignment slack
// TMEM columns: [0, 256) working region, [256, 512) momentum S.
//   working, tile t (hidden rows 128t..128t+127) at column 128t:
//     +0..63   Z_K^T, then silu'(Z_K)^T, then dW1_c
//     +64..127 Z_Q^T, then (GW2)^T, then dW2^T_c     (tile 0's +64..127 also hosts Y)
//   S region, tile t at column 256 + 128t: +0..63 S1 rows, +64..127 S2^T rows.
constexpr uint32_t kTmemCols = 512;
}  // namespace tc

static_assert(tc::kSmemBytes <= 232448, "shared memory budget");

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// Writes a 64-element fp32 row as bf16 into row `row` of a swizzled [rows][64] tile.
__device__ __forceinline__ void store_row_bf16(uint32_t tile, int row, const float (&w)[64]) {
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        const uint32_t a = tile + (uint32_t)row * 128u + ((uint32_t)(ch ^ (row & 7)) << 4);
        st_shared_v4(a, pack_bf16x2(w[8 * ch + 0], w[8 * ch + 1]), pack_bf16x2(w[8 * ch + 2], w[8 * ch + 3]),
                     pack_bf16x2(w[8 * ch + 4], w[8 * ch + 5]), pack_bf16x2(w[8 * ch + 6], w[8 * ch + 7]));
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

__device__ __forceinline__ float sigmoidf_fast(float z) { return __fdividef(1.f, 1.f + __expf(-z)); }

__global__ void __launch_bounds__(tc::kThreads, 1) chunk_fwd_tc_mlp64(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
    const __grid_constant__ CUtensorMap tmV, const float* __restrict__ alpha, const float* __restrict__ eta,
    const float* __restrict__ theta, float* __restrict__ W1g, float* __restrict__ W2g, float* __restrict__ S1g,
    float* __restrict__ S2g, __nv_bfloat16* __restrict__ yg, long T, int chunk, unsigned* status) {
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    float* s_alpha = reinterpret_cast<float*>(sm + ALPHA);
    float* s_eta = reinterpret_cast<float*>(sm + ETA);
    float* s_theta = reinterpret_cast<float*>(sm + THETA);
    float* s_c = reinterpret_cast<float*>(sm + CC);
    float* s_d = reinterpret_cast<float*>(sm + DD);
    float* s_scal = reinterpret_cast<float*>(sm + SCAL);
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + BAR);
    uint64_t* bar_mma = bar_tma + 2;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + FLAG);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int hrow = half * 128 + quad * 32 + lane;  // hidden row owned by this thread
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const long u = blockIdx.x;

    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmV);
    }
    if (warp == 0) {
        tmem_alloc(reinterpret_cast<uint32_t*>(sm + TPTR), kTmemCols);
        tmem_relinquish();
    }
    // Token tiles start at zero: rows beyond the chunk length are never written by TMA.
    for (uint32_t o = tid * 16; o < 49152; o += kThreads * 16) st_shared_v4(sb + KQ0 + o, 0u, 0u, 0u, 0u);

    // State of this thread's hidden row.
    float w1[64], w2[64];
    {
        const float4* p = reinterpret_cast<const float4*>(W1g + (u * kH + hrow) * kD);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float4 x = p[i];
            w1[4 * i] = x.x;
            w1[4 * i + 1] = x.y;
            w1[4 * i + 2] = x.z;
            w1[4 * i + 3] = x.w;
        }
        const float* q2 = W2g + u * kD * kH + hrow;
#pragma unroll
        for (int i = 0; i < 64; ++i) w2[i] = q2[(size_t)i * kH];
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + TPTR);
    const uint32_t t_work = tmem + lane_off + half * 128;        // this warp's working columns
    const uint32_t t_s = tmem + lane_off + 256 + half * 128;     // S1 at +0, S2^T at +64
    {
        const float* p1 = S1g + (u * kH + hrow) * kD;
        const float* p2 = S2g + u * kD * kH + hrow;
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
            uint32_t r[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(p1[16 * hh + i]);
            tmem_st16(t_s + 16 * hh, r);
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(p2[(size_t)(16 * hh + i) * kH]);
            tmem_st16(t_s + 64 + 16 * hh, r);
        }
    }
    store_row_bf16(sb + W1, hrow, w1);
    store_row_bf16(sb + W2T, hrow, w2);
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int nchunks = (int)((T + chunk - 1) / chunk);
    const uint32_t tx_bytes = 3u * (uint32_t)chunk * 128u;
    uint32_t tma_issued[2] = {0, 0}, tma_done[2] = {0, 0};  // used by thread 0 only
    auto issue_tma = [&](int c, int b) {
        const uint32_t kq = b ? KQ1 : KQ0, vv = b ? V1 : V0;
        mbar_arrive_expect_tx(&bar_tma[b], tx_bytes);
        tma_load_3d(sm + kq, &tmK, &bar_tma[b], 0, c * chunk, (int)u);
        tma_load_3d(sm + kq + 8192, &tmQ, &bar_tma[b], 0, c * chunk, (int)u);
        tma_load_3d(sm + vv, &tmV, &bar_tma[b], 0, c * chunk, (int)u);
        ++tma_issued[b];
    };
    if (tid == 0) {
        issue_tma(0, 0);
        if (nchunks > 1) issue_tma(1, 1);
    }
    uint32_t mma_phase = 0;
    bool mma_pending = false;  // thread 0: a commit not yet waited for
    auto wait_mma = [&]() {
        if (!mbar_wait(bar_mma, mma_phase)) {
            atomicOr(status, kStatusTimeoutMma);
            *abort_flag = 1;
        } else if (tid == 0) {
            mma_pending = false;
        }
        mma_phase ^= 1u;
        tc_fence_after();
    };

    const uint32_t idZ = idesc_bf16_f32(128, 128, 0, 0);
    const uint32_t idY = idesc_bf16_f32(128, 64, 1, 1);
    const uint32_t idG = idesc_bf16_f32(128, 64, 0, 0);
    const uint32_t idW = idesc_bf16_f32(128, 64, 0, 1);

    for (int c = 0; c < nchunks; ++c) {
        const int buf = c & 1;
        const uint32_t KQb = buf ? KQ1 : KQ0, Vb = buf ? V1 : V0;
        const long t0 = (long)c * chunk;
        const int n = (int)min((long)chunk, T - t0);

        // (A) gates; K, Q tiles landed -> Z^T = W1 [K;Q]^T
        if (tid < kN) {
            const long g = u * T + t0 + tid;
            s_alpha[tid] = tid < n ? alpha[g] : 0.f;
            s_eta[tid] = tid < n ? eta[g] : 1.f;
            s_theta[tid] = tid < n ? theta[g] : 0.f;
        }
        // Every thread waits on the tile barrier itself: the K and V tiles are read below
        // with ordinary shared-memory loads as well as by the MMAs.
        const bool landed = mbar_wait(&bar_tma[buf], (uint32_t)(c >> 1) & 1u);
        if (!landed) {
            atomicOr(status, kStatusTimeoutTma);
            *abort_flag = 1;
        }
        if (tid == 0) {
            if (landed) {
                ++tma_done[buf];
                tc_fence_after();
#pragma unroll
                for (int t = 0; t < 2; ++t)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(tmem + t * 128, sdesc_sw128(sb + W1 + t * 16384 + ks * 32, 16, 1024),
                                  sdesc_sw128(sb + KQb + ks * 32, 16, 1024), idZ, ks > 0);
                umma_commit(bar_mma);
                mma_pending = true;
            }
        }
        __syncthreads();
        if (*abort_flag) break;

        // (B) gate scan
        if (warp == 0) gate_scan(n, s_alpha, s_eta, s_theta, s_c, s_d, s_scal, lane);
        __syncthreads();

        // (C) momentum pre-pass: W <- A W + sigma S, S <- E S (the d-GEMM then adds -sum d_j g_j);
        //     scaled key tiles -c_t K[t], -d_t K[t]
        {
            const float An = s_scal[0], En = s_scal[1], sig = s_scal[2];
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
                uint32_t r[16];
                tmem_ld16(t_s + 16 * hh, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float s = __uint_as_float(r[i]);
                    w1[16 * hh + i] = An * w1[16 * hh + i] + sig * s;
                    r[i] = __float_as_uint(En * s);
                }
                tmem_st16(t_s + 16 * hh, r);
            }
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
                uint32_t r[16];
                tmem_ld16(t_s + 64 + 16 * hh, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float s = __uint_as_float(r[i]);
                    w2[16 * hh + i] = An * w2[16 * hh + i] + sig * s;
                    r[i] = __float_as_uint(En * s);
                }
                tmem_st16(t_s + 64 + 16 * hh, r);
            }
            for (int qc = tid; qc < 512; qc += kThreads) {  // 16-byte chunks of the K tile
                const uint32_t off = (uint32_t)qc * 16u;
                const int row = qc >> 3;
                const uint4 kv = ld_shared_v4(sb + KQb + off);
                const float cr = -s_c[row], dr = -s_d[row];
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
            tmem_wait_st();
        }
        wait_mma();  // Z^T ready

        // (D) A = silu(Z): keys -> AT0 (and silu'(Z_K) back into TMEM), queries -> AT1
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) {  // 16-column blocks: 0..3 keys, 4..7 queries
            uint32_t r[16];
            tmem_ld16(t_work + 16 * cb, r);
            tmem_wait_ld();
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                const float z0 = __uint_as_float(r[i]), z1 = __uint_as_float(r[i + 1]);
                const float s0 = sigmoidf_fast(z0), s1 = sigmoidf_fast(z1);
                pk[i / 2] = pack_bf16x2(z0 * s0, z1 * s1);
                r[i] = __float_as_uint(s0 * (1.f + z0 * (1.f - s0)));
                r[i + 1] = __float_as_uint(s1 * (1.f + z1 * (1.f - s1)));
            }
            const uint32_t tile = (cb < 4 ? AT0 : AT1), ch0 = (cb & 3) * 2;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                const uint32_t addr = sb + tile + (uint32_t)hrow * 128u + ((uint32_t)((ch0 + ch) ^ (hrow & 7)) << 4);
                st_shared_v4(addr, pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
            }
            if (cb < 4) tmem_st16(t_work + 16 * cb, r);
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;

        // (E) Y = A W2^T for keys (rows 0..63) and queries (rows 64..127) -> TMEM cols 64..127
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 16; ++ks)
                umma_bf16(tmem + 64, sdesc_sw128(sb + AT0 + ks * 2048, AT1 - AT0, 1024),
                          sdesc_sw128(sb + W2T + ks * 2048, 8192, 1024), idY, ks > 0);
            umma_commit(bar_mma);
            mma_pending = true;
        }
        wait_mma();

        // (F) keys: G = 2 (M(k) - v) and its scaled copies; queries: y
        {
            const int row = quad * 32 + lane;  // TMEM lane = token row of Y
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                const int col0 = half * 32 + 16 * hb;
                uint32_t r[16];
                tmem_ld16(tmem + lane_off + 64 + col0, r);
                tmem_wait_ld();
                if (row < kN) {
                    const float cr = -s_c[row], dr = -s_d[row];
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch) {
                        const uint32_t off = sw128_off((uint32_t)row, (uint32_t)(col0 + 8 * ch));
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
                } else if (row - kN < n) {
                    uint4* dst = reinterpret_cast<uint4*>(yg + ((u * T + t0 + (row - kN)) * kD + col0));
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch) {
                        uint4 o;
                        o.x = pack_bf16x2(__uint_as_float(r[8 * ch]), __uint_as_float(r[8 * ch + 1]));
                        o.y = pack_bf16x2(__uint_as_float(r[8 * ch + 2]), __uint_as_float(r[8 * ch + 3]));
                        o.z = pack_bf16x2(__uint_as_float(r[8 * ch + 4]), __uint_as_float(r[8 * ch + 5]));
                        o.w = pack_bf16x2(__uint_as_float(r[8 * ch + 6]), __uint_as_float(r[8 * ch + 7]));
                        dst[ch] = o;
                    }
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;

        // (G) (GW2)^T = W2^T G^T -> tile t cols 128t+64..; S2^T += A_K^T diag(-d) G
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(tmem + t * 128 + 64, sdesc_sw128(sb + W2T + t * 16384 + ks * 32, 16, 1024),
                              sdesc_sw128(sb + G + ks * 32, 16, 1024), idG, ks > 0);
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(tmem + 256 + t * 128 + 64, sdesc_sw128(sb + AT0 + t * 16384 + ks * 32, 16, 1024),
                              sdesc_sw128(sb + GD + ks * 2048, 8192, 1024), idW, 1);
            umma_commit(bar_mma);
            mma_pending = true;
        }
        wait_mma();

        // (H) Delta^T = (GW2)^T * silu'(Z_K)^T -> AT1 (the queries' tile is no longer needed)
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            uint32_t g[16], s[16];
            tmem_ld16(t_work + 64 + 16 * cb, g);
            tmem_ld16(t_work + 16 * cb, s);
            tmem_wait_ld();
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                const uint32_t addr =
                    sb + AT1 + (uint32_t)hrow * 128u + ((uint32_t)((2 * cb + ch) ^ (hrow & 7)) << 4);
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(g[8 * ch + e]) * __uint_as_float(s[8 * ch + e]);
                st_shared_v4(addr, pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                             pack_bf16x2(x[6], x[7]));
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;

        // (I) dW1_c' -> cols 128t, S1 += Delta^T diag(-d) K, dW2^T_c' -> cols 128t+64; prefetch chunk c+2
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t dA = sdesc_sw128(sb + AT1 + t * 16384 + ks * 32, 16, 1024);
                    const uint64_t aA = sdesc_sw128(sb + AT0 + t * 16384 + ks * 32, 16, 1024);
                    umma_bf16(tmem + t * 128, dA, sdesc_sw128(sb + KC + ks * 2048, 8192, 1024), idW, ks > 0);
                    umma_bf16(tmem + 256 + t * 128, dA, sdesc_sw128(sb + KD + ks * 2048, 8192, 1024), idW, 1);
                    umma_bf16(tmem + t * 128 + 64, aA, sdesc_sw128(sb + GC + ks * 2048, 8192, 1024), idW, ks > 0);
                }
            umma_commit(bar_mma);
            mma_pending = true;
            if (c + 2 < nchunks) issue_tma(c + 2, buf);
        }
        wait_mma();

        // (J) W <- (A W + sigma S) - sum_j c_j g_j; refresh the bf16 operand copies
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            uint32_t r1[16], r2[16];
            tmem_ld16(t_work + 16 * cb, r1);
            tmem_ld16(t_work + 64 + 16 * cb, r2);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                w1[16 * cb + i] += __uint_as_float(r1[i]);
                w2[16 * cb + i] += __uint_as_float(r2[i]);
            }
        }
        store_row_bf16(sb + W1, hrow, w1);
        store_row_bf16(sb + W2T, hrow, w2);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;
    }

    // Drain (only after an abort can copies or MMAs still be in flight), then write the state.
    if (tid == 0) {
        for (int b = 0; b < 2; ++b)
            while (tma_done[b] < tma_issued[b]) {
                if (!mbar_wait(&bar_tma[b], tma_done[b] & 1u)) break;
                ++tma_done[b];
            }
        if (mma_pending) mbar_wait(bar_mma, mma_phase);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    {
        float4* p = reinterpret_cast<float4*>(W1g + (u * kH + hrow) * kD);
#pragma unroll
        for (int i = 0; i < 16; ++i) p[i] = make_float4(w1[4 * i], w1[4 * i + 1], w1[4 * i + 2], w1[4 * i + 3]);
        float* q2 = W2g + u * kD * kH + hrow;
#pragma unroll
        for (int i = 0; i < 64; ++i) q2[(size_t)i * kH] = w2[i];
        float* p1 = S1g + (u * kH + hrow) * kD;
        float* p2 = S2g + u * kD * kH + hrow;
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
            uint32_t r[16];
            tmem_ld16(t_s + 16 * hh, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) p1[16 * hh + i] = __uint_as_float(r[i]);
            tmem_ld16(t_s + 64 + 16 * hh, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) p2[(size_t)(16 * hh + i) * kH] = __uint_as_float(r[i]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

size_t chunk_tc_mlp64_smem_bytes() { return tc::kSmemBytes; }

cudaError_t launch_chunk_tc_mlp64(const ForwardArgs& a, const CUtensorMap& tk, const CUtensorMap& tq,
                                  const CUtensorMap& tv, cudaStream_t st) {
    static bool attr_set = false;  // per process; the attribute is per function, not per device
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(chunk_fwd_tc_mlp64, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)tc::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    chunk_fwd_tc_mlp64<<<(unsigned)a.units, tc::kThreads, tc::kSmemBytes, st>>>(
        tk, tq, tv, a.alpha, a.eta, a.theta, a.W1, a.W2, a.S1, a.S2, (__nv_bfloat16*)a.y, a.T, a.chunk, a.status);
    return cudaGetLastError();
}

}  // namespace titans
