// Single-token decode step of the MLP memory (chunk = 1 semantics): y = M(q; W_{t-1}),
// g = grad ||M(k) - v||^2 at W_{t-1}, S <- eta S - theta g, W <- (1 - alpha) W + S
// ("Titans: Learning to Memorize at Test Time", walk-through sec. 3.1).
//
// The step reads and writes every state element once, so it is bound by HBM. One
// thread-block cluster per unit splits the hidden width into 64-row slices (C = h / 64
// CTAs): each CTA keeps its slice of W1 (64 x d) and W2 (d x 64) in registers, computes
// its partial M(k) and M(q), and the partials are summed across the cluster through
// distributed shared memory. The momentum slices S1, S2 are not needed before the update,
// so they stream into shared memory (cp.async) while the forward runs; that keeps the
// registers under 128 per thread and two CTAs resident per SM, so one CTA's loads overlap
// the other's arithmetic and cluster exchange. Every state element crosses HBM exactly
// twice (read, write).
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <atomic>

#include "kernels.h"

namespace cg = cooperative_groups;

namespace titans {

__device__ __forceinline__ float ld1(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld1(const __nv_bfloat16* p) { return __bfloat162float(*p); }

constexpr int kStepWarps = 8;
constexpr int kStepThreads = 32 * kStepWarps;
constexpr int kSlice = 64;  // hidden rows per CTA

// Dynamic shared memory of one CTA: the S1 slice [64][D] and S2 slice [D][64] (fp32).
template <int D>
constexpr size_t step_smem_bytes() {
    return (size_t)2 * kSlice * D * sizeof(float);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

template <int D, typename Tin>
__global__ void __launch_bounds__(kStepThreads, 2) step_mlp_cluster(
    const Tin* __restrict__ k, const Tin* __restrict__ q, const Tin* __restrict__ v,
    const float* __restrict__ alpha, const float* __restrict__ eta, const float* __restrict__ theta,
    float* __restrict__ W1, float* __restrict__ W2, float* __restrict__ S1, float* __restrict__ S2,
    Tin* __restrict__ y, const Tin* __restrict__ attn) {
    constexpr int H = 4 * D;
    constexpr int C = H / kSlice;        // CTAs per unit (cluster size)
    constexpr int MC = D / 32;           // W1 columns per lane
    constexpr int R1 = kSlice / kStepWarps;  // W1 rows per warp
    constexpr int R2 = D / kStepWarps;       // W2 rows per warp
    __shared__ float sk[D], sq[D], sv[D], sG[D];
    __shared__ float zk[kSlice], zq[kSlice], ak[kSlice], aq[kSlice], sp[kSlice], dl[kSlice];
    __shared__ float part[2][D];
    __shared__ float red[kStepWarps][kSlice];
    extern __shared__ float4 step_dyn[];
    float* sS1 = reinterpret_cast<float*>(step_dyn);  // [kSlice][D]
    float* sS2 = sS1 + kSlice * D;                    // [D][kSlice]

    cg::cluster_group cluster = cg::this_cluster();
    const int r = (int)cluster.block_rank();
    const long u = blockIdx.x / C;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j0 = r * kSlice;  // first hidden row of this slice

    const float* W1u = W1 + u * H * D;
    const float* S1u = S1 + u * H * D;
    const float* W2u = W2 + u * D * H;
    const float* S2u = S2 + u * D * H;

    // Issue every state load first: S1 and S2 slices into shared memory (16-byte pieces),
    // W1 and W2 slices into registers; the arithmetic below waits on them.
    {
        const float* src1 = S1u + (size_t)j0 * D;  // contiguous [kSlice][D]
#pragma unroll
        for (int m = 0; m < kSlice * D / 4 / kStepThreads; ++m) {
            const int id = tid + kStepThreads * m;
            cp_async16(sS1 + 4 * id, src1 + 4 * id);
        }
#pragma unroll
        for (int m = 0; m < D * kSlice / 4 / kStepThreads; ++m) {
            const int id = tid + kStepThreads * m, row = id / (kSlice / 4), q4 = id % (kSlice / 4);
            cp_async16(sS2 + row * kSlice + 4 * q4, S2u + (size_t)row * H + j0 + 4 * q4);
        }
    }
    float w1[R1][MC], w2[R2][2];
#pragma unroll
    for (int i = 0; i < R1; ++i)
#pragma unroll
        for (int c = 0; c < MC; ++c)
            w1[i][c] = __ldcs(W1u + (size_t)(j0 + warp * R1 + i) * D + lane + 32 * c);
#pragma unroll
    for (int i = 0; i < R2; ++i)
#pragma unroll
        for (int c = 0; c < 2; ++c) w2[i][c] = __ldcs(W2u + (size_t)(warp + kStepWarps * i) * H + j0 + lane + 32 * c);
    for (int i = tid; i < D; i += kStepThreads) {
        sk[i] = ld1(k + u * D + i);
        sq[i] = ld1(q + u * D + i);
        sv[i] = ld1(v + u * D + i);
    }
    const float al = alpha[u], et = eta[u], th = theta[u];
    __syncthreads();

    // z = W1 k and W1 q for this slice: one warp-reduction per row.
#pragma unroll
    for (int i = 0; i < R1; ++i) {
        float a = 0.f, b = 0.f;
#pragma unroll
        for (int c = 0; c < MC; ++c) {
            a += w1[i][c] * sk[lane + 32 * c];
            b += w1[i][c] * sq[lane + 32 * c];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            a += __shfl_xor_sync(0xffffffffu, a, o);
            b += __shfl_xor_sync(0xffffffffu, b, o);
        }
        if (lane == 0) {
            zk[warp * R1 + i] = a;
            zq[warp * R1 + i] = b;
        }
    }
    __syncthreads();
    if (tid < kSlice) {
        const float z = zk[tid], s = 1.f / (1.f + expf(-z));
        ak[tid] = z * s;
        sp[tid] = s * (1.f + z * (1.f - s));
        const float zz = zq[tid];
        aq[tid] = zz / (1.f + expf(-zz));
    }
    __syncthreads();
    // Partial W2 silu(.) over this slice's 64 hidden units.
#pragma unroll
    for (int i = 0; i < R2; ++i) {
        float a = w2[i][0] * ak[lane] + w2[i][1] * ak[lane + 32];
        float b = w2[i][0] * aq[lane] + w2[i][1] * aq[lane + 32];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            a += __shfl_xor_sync(0xffffffffu, a, o);
            b += __shfl_xor_sync(0xffffffffu, b, o);
        }
        if (lane == 0) {
            part[0][warp + kStepWarps * i] = a;
            part[1][warp + kStepWarps * i] = b;
        }
    }
    cluster.sync();
    // Sum the partials of all C slices (distributed shared memory), in rank order.
    for (int i = tid; i < D; i += kStepThreads) {
        float yh = 0.f, yq = 0.f;
#pragma unroll
        for (int rr = 0; rr < C; ++rr) {
            const float* pr = cluster.map_shared_rank(&part[0][0], rr);
            yh += pr[i];
            yq += pr[D + i];
        }
        sG[i] = 2.f * (yh - sv[i]);
        if (r == 0) {
            // the retrieval, or the memory-as-a-gate output attn * sigmoid(M(q))
            const float o = attn ? ld1(attn + u * D + i) * (1.f / (1.f + expf(-yq))) : yq;
            if constexpr (sizeof(Tin) == 2)
                y[u * D + i] = __float2bfloat16_rn(o);
            else
                y[u * D + i] = o;
        }
    }
    // This CTA is done reading the other slices' partials: arrive now, wait only before
    // exiting, so no CTA holds its SM until the slowest one of the cluster has stored.
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    __syncthreads();
    // Backprop through W2 for this slice's hidden units: per-lane partial over its rows.
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < R2; ++i) acc += w2[i][c] * sG[warp + kStepWarps * i];
        red[warp][lane + 32 * c] = acc;
    }
    __syncthreads();
    if (tid < kSlice) {
        float b = 0.f;
#pragma unroll
        for (int w = 0; w < kStepWarps; ++w) b += red[w][tid];
        dl[tid] = b * sp[tid];
    }
    cp_async_wait_all();
    __syncthreads();
    float* W1w = W1 + u * H * D;
    float* S1w = S1 + u * H * D;
    float* W2w = W2 + u * D * H;
    float* S2w = S2 + u * D * H;
#pragma unroll
    for (int i = 0; i < R1; ++i)
#pragma unroll
        for (int c = 0; c < MC; ++c) {
            const int jl = warp * R1 + i, m = lane + 32 * c;
            const size_t o = (size_t)(j0 + jl) * D + m;
            const float s = et * sS1[jl * D + m] - th * (dl[jl] * sk[m]);
            __stcs(S1w + o, s);
            __stcs(W1w + o, (1.f - al) * w1[i][c] + s);
        }
#pragma unroll
    for (int i = 0; i < R2; ++i)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int row = warp + kStepWarps * i, jj = lane + 32 * c;
            const size_t o = (size_t)row * H + j0 + jj;
            const float s = et * sS2[row * kSlice + jj] - th * (sG[row] * ak[jj]);
            __stcs(S2w + o, s);
            __stcs(W2w + o, (1.f - al) * w2[i][c] + s);
        }
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");  // no CTA leaves while another may still read its partials
}

template <int D, typename Tin>
static cudaError_t launch_step(const ForwardArgs& a, cudaStream_t st) {
    constexpr int C = 4 * D / kSlice;
    // The shared-memory opt-in is per function and device: set it once per device.
    static std::atomic<unsigned long long> attr_set{0};
    int dev = 0;
    cudaError_t e0 = cudaGetDevice(&dev);
    if (e0 != cudaSuccess) return e0;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(attr_set.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(step_mlp_cluster<D, Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)step_smem_bytes<D>());
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(bit);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.units * C));
    cfg.blockDim = dim3(kStepThreads);
    cfg.dynamicSmemBytes = step_smem_bytes<D>();
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, step_mlp_cluster<D, Tin>, (const Tin*)a.k, (const Tin*)a.q, (const Tin*)a.v,
                              a.alpha, a.eta, a.theta, a.W1, a.W2, a.S1, a.S2, (Tin*)a.y, (const Tin*)a.attn);
}

cudaError_t launch_step_cluster(const ForwardArgs& a, cudaStream_t st) {
    if (a.d == 64) return a.bf16 ? launch_step<64, __nv_bfloat16>(a, st) : launch_step<64, float>(a, st);
    if (a.d == 128) return a.bf16 ? launch_step<128, __nv_bfloat16>(a, st) : launch_step<128, float>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace titans
