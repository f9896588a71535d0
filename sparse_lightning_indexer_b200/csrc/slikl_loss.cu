// Per-token KL loss output (optional): L_t = sum over the valid slots j with p_j > 0 of
// p_j log(p_j / y_j), the loss whose gradient the operator computes
// (aclnnSparseLightningIndexerKLLossGrad, section "计算公式": the KL divergence between the
// target distribution p = attnSoftmaxL1Norm and y = Softmax(I)).
//
// It reads y back from softmax_out, which the fused kernel has just written, with p and the
// indices: one warp per query row, lanes over the slots, a fixed-order warp reduction (the
// result is bitwise reproducible). A slot is valid when its index lies in [0, key count of the
// row's batch), the same test as the fused kernel's. y is clamped below at the smallest normal
// fp32 value, so a y that underflowed to 0 gives a large finite term instead of infinity.
#include <float.h>

#include "slikl_common.cuh"

namespace slikl {
namespace {

__global__ void kl_loss(Params P, float *loss) {
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= P.T1) return;
    const int32_t kl = P.tok_klen[t];
    const int64_t ro = t * (int64_t)P.K;
    float acc = 0.f;
    for (int j = lane; j < P.K; j += 32) {
        const int32_t v = P.idx[ro + j];
        const float pj = P.p[ro + j];
        if (v >= 0 && v < kl && pj > 0.f) {
            const float yj = fmaxf(P.y[ro + j], FLT_MIN);
            acc += pj * (logf(pj) - logf(yj));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) loss[t] = acc;
}

}  // namespace

cudaError_t launch_kl_loss(const Params &P, float *loss, cudaStream_t s) {
    if (P.T1 <= 0) return cudaSuccess;
    const int64_t blocks = (P.T1 * 32 + 255) / 256;
    kl_loss<<<(unsigned)blocks, 256, 0, s>>>(P, loss);
    return cudaGetLastError();
}

}  // namespace slikl
