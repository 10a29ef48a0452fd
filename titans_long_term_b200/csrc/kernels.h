// Host-side launch interface shared by the library's .cu files (not part of the C ABI).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>

namespace titans {

struct ForwardArgs {
    int d, h;          // h = 0: linear memory
    long units, T;
    int chunk;
    bool bf16;         // k, q, v, y dtype
    const void *k, *q, *v;
    const float *alpha, *eta, *theta;
    long gate_ld;      // elements between consecutive units' gate rows (T for [B, H, T])
    bool chunk_gates;  // gates shared by a chunk's tokens: [units][ceil(T / chunk)], token t reads t / chunk
    float *W1, *W2, *S1, *S2;
    void* y;
    const void* attn;  // NULL: y = M(q); else y = attn * sigmoid(M(q)) (memory-as-a-gate output), dtype of y
    float* ws;         // CUDA-core path workspace
    size_t ws_per_unit;
    unsigned* status;  // device status word
    // Tensor-core chunk kernel only: when set, every chunk's start state [W1 | W2 | S1 | S2] (fp32,
    // 4 h d floats) is also written to ckpt + unit * ckpt_unit_stride + chunk * 4 h d.
    float* ckpt = nullptr;
    size_t ckpt_unit_stride = 0;
};

size_t cuda_cores_ws_floats(int d, int h, int n);
cudaError_t launch_chunk_cuda_cores(const ForwardArgs& a, cudaStream_t st);
// Loads both instantiations (fp32 and bf16 inputs) of the CUDA-core kernel on the current device.
cudaError_t preload_chunk_cuda_cores();
cudaError_t launch_step_cluster(const ForwardArgs& a, cudaStream_t st);
// Tensor-core chunk kernel (d = 64, h = 256, chunk <= 64, bf16). The tensor maps
// describe k, q, v as [units][T][64] bf16 with a {64, chunk, 1} box and 128-byte swizzle.
cudaError_t launch_chunk_tc_mlp64(const ForwardArgs& a, const CUtensorMap& tk, const CUtensorMap& tq,
                                  const CUtensorMap& tv, cudaStream_t st);
size_t chunk_tc_mlp64_smem_bytes();
// Both SiLU evaluations of the chunk kernel (FMA-pipe and special-function-unit tanh) on n values.
cudaError_t launch_silu_routes(const float* h, float* s_fma, float* s_mufu, long n, cudaStream_t st);
// Phased tensor-core chunk kernel of the wide memory (d = 128, h = 512, chunk <= 128, bf16): a
// cooperative persistent launch over all SMs. Needs tc_phased_ws_bytes_per_unit() bytes of
// workspace per unit (a.ws, a.ws_per_unit floats apart) and two device words `sync` for its grid
// barrier (zeroed by the launch itself).
// Deep memory (L >= 2 layers, packed state W, S [units][deep_state_floats] in ForwardArgs::W1 / S1),
// CUDA-core chunk kernel; workspace deep_ws_floats per unit.
size_t deep_ws_floats(int d, int h, int layers, int n);
__host__ __device__ size_t deep_state_floats(int d, int h, int layers);
cudaError_t launch_chunk_deep_cuda_cores(const ForwardArgs& a, int layers, cudaStream_t st);
// Tensor-core chunk kernel of the deep memory (bf16, d in {64, 128}, h = 4d, 3..8 layers, chunk <= 128):
// phased cooperative launch over all SMs like the wide 2-layer kernel; needs
// tc_deep_ws_bytes_per_unit() bytes of workspace per unit and the two grid-barrier words `sync`.
size_t tc_deep_ws_bytes_per_unit(int d, int h, int layers);
bool tc_deep_supported(int d, int h, int layers, int chunk);
cudaError_t launch_chunk_tc_deep(const ForwardArgs& a, int layers, unsigned* sync, cudaStream_t st);
// Linear memory by the cross-chunk scan: up to nseg_max segments per unit, each needing
// linear_scan_slot_floats(d, chunk) floats of workspace (a.ws, a.ws_per_unit floats per unit).
size_t linear_scan_slot_floats(int d, int n);
cudaError_t launch_linear_scan(const ForwardArgs& a, int nseg_max, cudaStream_t st);
// Backward of the chunked linear memory (see linear_backward.cu).
struct LinearBackwardArgs {
    int d, chunk;
    long units, T;
    bool bf16;
    const void *k, *q, *v, *dy;
    const float *alpha, *eta, *theta, *W0, *S0, *dWT, *dST;  // dWT, dST may be NULL (zero)
    void *dk, *dq, *dv;
    float *dalpha, *deta, *dtheta, *dW0, *dS0;
    float* ws;
    size_t ws_per_unit;  // floats
};
size_t linear_backward_ws_floats(int d, long T, int chunk);
// Backward of the chunked 2-layer MLP memory (see mlp_backward.cu).
struct MlpBackwardArgs {
    int d, h, chunk;
    long units, T;
    bool bf16;
    const void *k, *q, *v, *dy;
    const float *alpha, *eta, *theta;
    const float *W1, *W2, *S1, *S2;       // initial state
    const float *dW1, *dW2, *dS1, *dS2;   // upstream adjoints of the final state, NULL = zero
    void *dk, *dq, *dv;
    float *dalpha, *deta, *dtheta;
    float *dW1_0, *dW2_0, *dS1_0, *dS2_0;
    float* ws;
    size_t ws_per_unit;  // floats
    unsigned* status;    // device status word (the tensor-core backward's bounded waits)
    bool ckpt_ready = false;  // tensor-core backward: the chunk-start states are already in the workspace
};
size_t mlp_backward_ws_floats(int d, int h, long T, int chunk);
cudaError_t launch_mlp_backward(const MlpBackwardArgs& a, cudaStream_t st);
// Tensor-core backward of the 2-layer memory (bf16, d = 64, h = 256, chunk <= 64): one CTA per unit,
// mlp_backward_tc_ws_bytes() of workspace per unit (MlpBackwardArgs::ws_per_unit floats apart).
bool mlp_backward_tc_supported(int d, int h, int chunk);
size_t mlp_backward_tc_ws_bytes(long T, int chunk);
size_t mlp_backward_tc_ckpt_offset();  // byte offset of the chunk-start states in a unit's workspace
cudaError_t launch_mlp_backward_tc(const MlpBackwardArgs& a, cudaStream_t st);
cudaError_t launch_linear_backward(const LinearBackwardArgs& b, cudaStream_t st);
size_t tc_phased_ws_bytes_per_unit();
bool tc_phased_supported(int d, int h, int chunk);
cudaError_t launch_chunk_tc_phased(const ForwardArgs& a, unsigned* sync, cudaStream_t st);

}  // namespace titans
