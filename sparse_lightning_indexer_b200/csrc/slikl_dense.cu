// Dense variant: the index rows that turn DenseLightningIndexerKLLossGrad into the sparse
// operator's problem (reading in include/slikl.h: slot j of a row is key j of its batch, the
// first L_t of them visible under the mask). One warp per query row writes 0, 1, .., L_t - 1
// and then -1 up to the row length; the sparse kernels then run unchanged.
#include "slikl_common.cuh"

namespace slikl {
namespace {

struct DenseArgs {
    int32_t *idx;          // [T1][Ld]
    int64_t T1, B, S1, S2;
    int Ld, layout_q, layout_k, mask;
    const int32_t *cu_q, *cu_k, *used_q, *used_k;
    uint32_t *flag;        // SLIKL_DEV_ROW_LEN_BELOW_KEYS when a batch has more keys than Ld
};

// Largest b in [0, B) with cu[b] <= t (binary search; stays in range for any array contents).
__device__ int64_t batch_of_row(const int32_t *cu, int64_t B, int64_t t) {
    int64_t lo = 0, hi = B - 1;
    while (lo < hi) {
        const int64_t mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ int64_t clamp_len(int64_t v, int64_t hi) { return v < 0 ? 0 : (v > hi ? hi : v); }

__global__ void dense_indices(DenseArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t wpb = blockDim.x >> 5;
    for (int64_t t = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5); t < a.T1;
         t += (int64_t)gridDim.x * wpb) {
        int64_t b, q0, qlen, klen;
        if (a.layout_q == SLIKL_BSND) {
            b = t / a.S1;
            q0 = b * a.S1;
            qlen = a.S1;
        } else {
            b = batch_of_row(a.cu_q, a.B, t);
            q0 = a.cu_q[b];
            qlen = clamp_len((int64_t)a.cu_q[b + 1] - q0, a.T1);
        }
        klen = a.layout_k == SLIKL_BSND ? a.S2 : clamp_len((int64_t)a.cu_k[b + 1] - a.cu_k[b], 1ll << 31);
        if (a.used_q) qlen = clamp_len(a.used_q[b], qlen);
        if (a.used_k) klen = clamp_len(a.used_k[b], klen);
        const int64_t s = t - q0;
        int64_t L = 0;
        if (s >= 0 && s < qlen) L = clamp_len(a.mask == 0 ? klen : s + klen - qlen + 1, klen);
        if (L > a.Ld) {
            if (lane == 0) atomicOr(a.flag, SLIKL_DEV_ROW_LEN_BELOW_KEYS);
            L = a.Ld;
        }
        int32_t *row = a.idx + t * a.Ld;
        for (int j = lane; j < a.Ld; j += 32) row[j] = j < L ? j : -1;
    }
}

__global__ void dense_flag_merge(const uint32_t *flag, uint32_t *status) {
    if (threadIdx.x == 0 && *flag) atomicOr(status, *flag);
}

}  // namespace

cudaError_t launch_dense_indices(int32_t *idx, int64_t T1, int64_t B, int64_t S1, int64_t S2,
                                 int Ld, int layout_q, int layout_k, int mask,
                                 const int32_t *cu_q, const int32_t *cu_k, const int32_t *used_q,
                                 const int32_t *used_k, uint32_t *flag, cudaStream_t s) {
    if (T1 <= 0) return cudaSuccess;
    DenseArgs a{idx, T1, B, S1, S2, Ld, layout_q, layout_k, mask, cu_q, cu_k, used_q, used_k, flag};
    const int64_t blocks = (T1 + 7) / 8;
    dense_indices<<<(unsigned)(blocks < 65535 * 16 ? blocks : 65535 * 16), 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_dense_flag_merge(const uint32_t *flag, uint32_t *status, cudaStream_t s) {
    dense_flag_merge<<<1, 32, 0, s>>>(flag, status);
    return cudaGetLastError();
}

}  // namespace slikl
