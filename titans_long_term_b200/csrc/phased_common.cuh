// Shared-memory staging, cp.async operand tiles and the bounded grid barrier of the phased
// tensor-core kernels (256 threads per CTA, one persistent CTA per SM, cooperative launch).
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"

namespace titans {
namespace phc {

constexpr int kThreads = 256;  // 8 warps: warp w reads TMEM lane quadrant w % 4, column half w / 4
constexpr unsigned kStatusTimeoutGrid = 4u;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

// Copies `rows` rows of 64 bf16 (128 B) into a swizzled [rows][64] tile at shared address `tile`:
// row r comes from src + r * stride (bytes). Rows r >= valid are zero.
__device__ __forceinline__ void load_tile(uint32_t tile, const uint8_t* src, size_t stride, int rows, int valid) {
    for (int i = threadIdx.x; i < rows * 8; i += kThreads) {
        const int r = i >> 3, c16 = i & 7;
        const uint32_t dst = tile + (uint32_t)r * 128u + ((uint32_t)(c16 ^ (r & 7)) << 4);
        if (r < valid)
            cp_async16(dst, src + (size_t)r * stride + (size_t)c16 * 16);
        else
            st_shared_v4(dst, 0u, 0u, 0u, 0u);
    }
}

// Byte offset of 16-byte chunk c of row r in a tile staged in shared memory with rows of `rb`
// bytes (a multiple of 128): within each group of eight chunks the index is XORed with r % 8, so
// that the 32 lanes of a warp, one row each, spread their 16-byte accesses over all banks, while a
// row's chunks stay inside the row.
__device__ __forceinline__ uint32_t srow_off(int r, int c, uint32_t rb) {
    return (uint32_t)r * rb + ((uint32_t)((c & ~7) | ((c ^ r) & 7)) << 4);
}
__device__ __forceinline__ uint32_t stage_off(int r, int c) { return srow_off(r, c, 512); }

// Coalesced copy of `rows` rows of rb bytes (row r at src + r * ld bytes) into the staged layout.
__device__ __forceinline__ void stage_rows_in(uint32_t tile, const void* src, size_t ld, int rows, uint32_t rb) {
    const int cpr = (int)(rb >> 4);
    for (int i = threadIdx.x; i < rows * cpr; i += kThreads) {
        const int r = i / cpr, c = i % cpr;
        cp_async16(tile + srow_off(r, c, rb), reinterpret_cast<const uint8_t*>(src) + (size_t)r * ld + 16 * c);
    }
}

// Coalesced copy of the first `rows` staged rows of rb bytes out to dst + r * ld bytes (L2 only):
// consecutive threads write consecutive 16-byte pieces of a row.
__device__ __forceinline__ void stage_rows_out(const uint8_t* tile, void* dst, size_t ld, int rows, uint32_t rb) {
    const int cpr = (int)(rb >> 4);
    for (int i = threadIdx.x; i < rows * cpr; i += kThreads) {
        const int r = i / cpr, c = i % cpr;
        __stcg(reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(dst) + (size_t)r * ld) + c,
               *reinterpret_cast<const uint4*>(tile + srow_off(r, c, rb)));
    }
}

// Coalesced copy of a [128 rows][128 floats] tile (row r at src + r * ld floats) into the staging layout.
__device__ __forceinline__ void stage_in(uint32_t tile, const float* src, size_t ld) {
    stage_rows_in(tile, src, ld * sizeof(float), 128, 512);
}

// All operand copies of the tile have landed and are visible to the tensor core.
__device__ __forceinline__ void operands_ready() {
    cp_async_wait_all();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
}

__device__ __forceinline__ uint32_t pack2(float a, float b) { return pack_bf16x2(a, b); }

// tanh via the hardware approximation (one MUFU op, relative error about 2^-11).
__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Grid-wide barrier with a bounded spin on sync[0] (arrivals; zero at launch); sync[1] is the abort
// flag. Returns false if any CTA gave up (a timeout anywhere). The kernel is launched cooperatively,
// so all CTAs are resident together.
__device__ __forceinline__ bool grid_sync(unsigned* sync, unsigned* status, unsigned& epoch, volatile uint32_t* s_ok) {
    __syncthreads();
    if (threadIdx.x == 0) {
        ++epoch;
        bool ok = true;
        __threadfence();
        atomicAdd(&sync[0], 1u);
        const unsigned target = epoch * gridDim.x;
        const unsigned long long t0 = globaltimer_ns();
        // Every CTA polls the same word: back off between polls so that the spinning CTAs do not
        // flood the L2 slice that holds it (the other CTAs' traffic goes through the same slices).
        for (unsigned it = 0;; ++it) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(&sync[0]) : "memory");
            if (v >= target) break;
            __nanosleep(128);
            if ((it & 15u) != 15u) continue;
            unsigned ab;
            asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(ab) : "l"(&sync[1]) : "memory");
            if (ab) {
                ok = false;
                break;
            }
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                atomicOr(status, kStatusTimeoutGrid);
                atomicExch(&sync[1], 1u);
                ok = false;
                break;
            }
        }
        __threadfence();
        *s_ok = ok ? 1u : 0u;
    }
    __syncthreads();
    return *s_ok != 0;
}

// Operand copies into the 128-byte-swizzled layouts the MMA descriptors describe.
//   K-major: element (r, k) at src[r * ld + k]; per 64-element K block kb a [R][64] tile at
//            dst + kb * R * 128; rows r >= valid_r are zero.
//   MN-major: element (r, k) at src[k * ld + r]; per 64-element K block kb and 64-element R block rb
//            a [64 k][64 r] tile at dst + (kb * R / 64 + rb) * 8192; K rows k >= valid_k are zero.
__device__ __forceinline__ void load_kmajor(uint32_t dst, const __nv_bfloat16* src, size_t ld, int R, int valid_r,
                                            int k0, int kc) {
    for (int kb = 0; kb < kc / 64; ++kb)
        load_tile(dst + (uint32_t)(kb * R * 128), reinterpret_cast<const uint8_t*>(src + k0 + kb * 64), ld * 2, R,
                  valid_r);
}
__device__ __forceinline__ void load_mnmajor(uint32_t dst, const __nv_bfloat16* src, size_t ld, int R, int k0,
                                             int kc, int valid_k) {
    for (int kb = 0; kb < kc / 64; ++kb)
        for (int rb = 0; rb < R / 64; ++rb)
            load_tile(dst + (uint32_t)((kb * (R / 64) + rb) * 8192),
                      reinterpret_cast<const uint8_t*>(src + (size_t)(k0 + kb * 64) * ld + rb * 64), ld * 2, 64,
                      valid_k - (k0 + kb * 64));
}
// Descriptor of K-step ks (16 elements) of an operand loaded by the functions above.
__device__ __forceinline__ uint64_t desc_k(uint32_t base, int R, int ks) {
    return sdesc_sw128(base + (uint32_t)((ks >> 2) * R * 128 + (ks & 3) * 32), 16, 1024);
}
__device__ __forceinline__ uint64_t desc_mn(uint32_t base, int R, int ks) {
    return sdesc_sw128(base + (uint32_t)((ks >> 2) * (R / 64) * 8192 + (ks & 3) * 2048), 8192, 1024);
}

__device__ __forceinline__ void mma_steps(uint32_t d_tmem, uint32_t a, bool a_mn, uint32_t b, bool b_mn, int N,
                                          int ksteps, bool acc) {
    const uint32_t id = idesc_bf16_f32(128, N, a_mn ? 1 : 0, b_mn ? 1 : 0);
    for (int ks = 0; ks < ksteps; ++ks)
        umma_bf16(d_tmem, a_mn ? desc_mn(a, 128, ks) : desc_k(a, 128, ks), b_mn ? desc_mn(b, N, ks) : desc_k(b, N, ks),
                  id, (acc || ks > 0) ? 1u : 0u);
}

}  // namespace phc
}  // namespace titans
