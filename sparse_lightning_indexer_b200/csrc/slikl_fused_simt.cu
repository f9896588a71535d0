// Fused per-token kernel on the CUDA cores (fp32 FMA). Generic over N1 <= 128, D <= 128 and
// any topk; it is the baseline that the tensor-core kernel (slikl_fused_sm100.cu) replaces
// on its supported shapes.
//
// Computes, for every query token of the CTA's range (aclnnSparseLightningIndexerKLLossGrad,
// section "计算公式"):
//   pass 1, 32-slot chunks:  K rows gathered to smem, S = q K^T, I = w . ReLU(S)
//   softmax:                 y = Softmax(I) over valid slots -> softmax_out, dI = y - p
//   pass 2, 32-slot chunks:  S recomputed, dW += dI . ReLU(S), dS = dI * w * 1[S > 0],
//                            dq += dS . K, dK rows = dS^T . q scattered to the key rows
// Every sum runs in a fixed order; only the atomic dK scatter is order dependent.
#include "slikl_common.cuh"

namespace slikl {
namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 32;

struct SimtSmem {
    // offsets in floats within dynamic shared memory
    int qs, kc, sc, iall, wv, rows, red;
    int total_floats;
};

__host__ __device__ inline SimtSmem simt_smem(int N1, int D, int K) {
    SimtSmem s;
    int off = 0;
    s.qs = off;   off += N1 * D;                 // q_t in fp32 [N1][D]
    s.kc = off;   off += kChunk * (D + 1);       // chunk of K rows [32][D+1]
    s.sc = off;   off += N1 * (kChunk + 1);      // S / dS chunk [N1][33]
    s.iall = off; off += K;                      // I, then dI, of every slot
    s.wv = off;   off += N1;                     // w_t
    s.rows = off; off += kChunk;                 // key rows of the chunk (int32)
    s.red = off;  off += 64;                     // reduction scratch
    s.total_floats = off;
    return s;
}

__device__ float block_reduce_max(float v, float *red) {
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float r = -INFINITY;
    for (int i = 0; i < kThreads / 32; ++i) r = fmaxf(r, red[i]);
    return r;
}

// Fixed-order sum: each thread's partial, then warp tree, then warps in index order.
__device__ float block_reduce_sum(float v, float *red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float r = 0.f;
    for (int i = 0; i < kThreads / 32; ++i) r += red[i];
    return r;
}

__global__ void __launch_bounds__(kThreads, 1) fused_simt(Params P) {
    extern __shared__ float smem[];
    const int N1 = P.N1, D = P.D, K = P.K;
    const SimtSmem L = simt_smem(N1, D, K);
    float *qs = smem + L.qs, *kc = smem + L.kc, *sc = smem + L.sc, *iall = smem + L.iall;
    float *wv = smem + L.wv, *red = smem + L.red;
    int32_t *rows = reinterpret_cast<int32_t *>(smem + L.rows);
    const int tid = threadIdx.x;
    const int t0 = P.meta[kMetaHeader + 2 * blockIdx.x];
    const int t1 = P.meta[kMetaHeader + 2 * blockIdx.x + 1];
    const int ND = N1 * D;
    constexpr int kMaxAcc = 128 * 128 / kThreads;   // dq elements per thread (N1*D <= 16384)

    for (int t = t0; t < t1; ++t) {
        const int32_t kbase = P.tok_kbase[t], klen = P.tok_klen[t];
        const int32_t *irow = P.idx + (int64_t)t * K;
        for (int e = tid; e < ND; e += kThreads) qs[e] = load_as_float(P.q, (int64_t)t * ND + e, P.dtype);
        for (int h = tid; h < N1; h += kThreads) wv[h] = P.w[(int64_t)t * N1 + h];
        __syncthreads();

        // ---- pass 1: I for every slot ----
        for (int c0 = 0; c0 < K; c0 += kChunk) {
            if (tid < kChunk) {
                int j = c0 + tid;
                rows[tid] = j < K ? slot_row(irow[j], kbase, klen) : -1;
            }
            __syncthreads();
            int any = __syncthreads_or(tid < kChunk && rows[tid] >= 0);
            if (!any) {
                for (int j = c0 + tid; j < c0 + kChunk && j < K; j += kThreads) iall[j] = -INFINITY;
                __syncthreads();
                continue;
            }
            for (int e = tid; e < kChunk * D; e += kThreads) {
                int jj = e / D, d = e - jj * D;
                int32_t r = rows[jj];
                kc[jj * (D + 1) + d] = r >= 0 ? load_as_float(P.k, (int64_t)r * D + d, P.dtype) : 0.f;
            }
            __syncthreads();
            for (int pidx = tid; pidx < N1 * kChunk; pidx += kThreads) {
                int h = pidx / kChunk, jj = pidx - h * kChunk;
                const float *qh = qs + h * D, *kr = kc + jj * (D + 1);
                float s = 0.f;
                for (int d = 0; d < D; ++d) s = fmaf(qh[d], kr[d], s);
                sc[h * (kChunk + 1) + jj] = s;
            }
            __syncthreads();
            if (tid < kChunk && c0 + tid < K) {
                float I = -INFINITY;
                if (rows[tid] >= 0) {
                    I = 0.f;
                    for (int h = 0; h < N1; ++h) I = fmaf(wv[h], fmaxf(sc[h * (kChunk + 1) + tid], 0.f), I);
                }
                iall[c0 + tid] = I;
            }
            __syncthreads();
        }

        // ---- softmax over valid slots, y and dI ----
        float m = -INFINITY;
        for (int j = tid; j < K; j += kThreads) m = fmaxf(m, iall[j]);
        m = block_reduce_max(m, red);
        float z = 0.f;
        if (m > -INFINITY)
            for (int j = tid; j < K; j += kThreads) z += iall[j] > -INFINITY ? __expf(iall[j] - m) : 0.f;
        z = block_reduce_sum(z, red);
        const float inv_z = z > 0.f ? 1.f / z : 0.f;
        for (int j = tid; j < K; j += kThreads) {
            float I = iall[j];
            float y = I > -INFINITY ? __expf(I - m) * inv_z : 0.f;
            P.y[(int64_t)t * K + j] = y;
            iall[j] = I > -INFINITY ? y - P.p[(int64_t)t * K + j] : 0.f;   // dI
        }
        __syncthreads();

        // ---- pass 2: dW, dq, dK ----
        float acc[kMaxAcc];
#pragma unroll
        for (int i = 0; i < kMaxAcc; ++i) acc[i] = 0.f;
        float dw_acc = 0.f;
        for (int c0 = 0; c0 < K; c0 += kChunk) {
            if (tid < kChunk) {
                int j = c0 + tid;
                rows[tid] = j < K ? slot_row(irow[j], kbase, klen) : -1;
            }
            __syncthreads();
            int any = __syncthreads_or(tid < kChunk && rows[tid] >= 0);
            if (!any) continue;
            for (int e = tid; e < kChunk * D; e += kThreads) {
                int jj = e / D, d = e - jj * D;
                int32_t r = rows[jj];
                kc[jj * (D + 1) + d] = r >= 0 ? load_as_float(P.k, (int64_t)r * D + d, P.dtype) : 0.f;
            }
            __syncthreads();
            for (int pidx = tid; pidx < N1 * kChunk; pidx += kThreads) {
                int h = pidx / kChunk, jj = pidx - h * kChunk;
                const float *qh = qs + h * D, *kr = kc + jj * (D + 1);
                float s = 0.f;
                for (int d = 0; d < D; ++d) s = fmaf(qh[d], kr[d], s);
                sc[h * (kChunk + 1) + jj] = s;
            }
            __syncthreads();
            if (tid < N1) {       // dW_h += sum_jj dI_jj * ReLU(S_h,jj), in slot order
                for (int jj = 0; jj < kChunk; ++jj) {
                    if (rows[jj] >= 0)
                        dw_acc = fmaf(iall[c0 + jj], fmaxf(sc[tid * (kChunk + 1) + jj], 0.f), dw_acc);
                }
            }
            __syncthreads();
            for (int pidx = tid; pidx < N1 * kChunk; pidx += kThreads) {   // S -> dS
                int h = pidx / kChunk, jj = pidx - h * kChunk;
                float s = sc[h * (kChunk + 1) + jj];
                sc[h * (kChunk + 1) + jj] = (rows[jj] >= 0 && s > 0.f) ? iall[c0 + jj] * wv[h] : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int i = 0; i < kMaxAcc; ++i) {      // dq += dS . K
                int e = tid + i * kThreads;
                if (e < ND) {
                    int h = e / D, d = e - h * D;
                    float a = acc[i];
                    for (int jj = 0; jj < kChunk; ++jj)
                        a = fmaf(sc[h * (kChunk + 1) + jj], kc[jj * (D + 1) + d], a);
                    acc[i] = a;
                }
            }
            for (int e = tid; e < kChunk * D; e += kThreads) {   // dK rows = dS^T . q
                int jj = e / D, d = e - jj * D;
                int32_t r = rows[jj];
                if (r < 0) continue;
                float v = 0.f;
                for (int h = 0; h < N1; ++h) v = fmaf(sc[h * (kChunk + 1) + jj], qs[h * D + d], v);
                if (P.deterministic)
                    P.partials[((int64_t)t * K + c0 + jj) * D + d] = v;
                else
                    red_add_f32(P.dk_acc + (int64_t)r * D + d, v);
            }
            __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < kMaxAcc; ++i) {
            int e = tid + i * kThreads;
            if (e < ND) store_from_float(P.dq, (int64_t)t * ND + e, acc[i], P.dtype);
        }
        if (tid < N1) P.dw[(int64_t)t * N1 + tid] = dw_acc;
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_fused_simt(const Params &P, int workers, cudaStream_t s) {
    const SimtSmem L = simt_smem(P.N1, P.D, P.K);
    size_t bytes = sizeof(float) * (size_t)L.total_floats;
    cudaError_t e = cudaFuncSetAttribute(fused_simt, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    fused_simt<<<workers, kThreads, bytes, s>>>(P);
    return cudaGetLastError();
}

}  // namespace slikl
