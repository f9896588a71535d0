// Work split ("metadata") of the merged B*S1 query rows over the CTAs of the fused kernel.
//
// The analogue of the DenseLightningIndexerKLLossGradMetadata AICPU operator (article on
// that operator, sections "功能定位" and "Metadata 输出布局"): there the merged rows are cut
// into formerCoreSize = ceil(total / cores) and remainCoreSize = formerCoreSize - 1 pieces.
// Here the split runs on the device, next to the data, and can also balance a per-row cost
// (mode 1) because the cost of a query row grows with its number of non-empty slot tiles.
//
// Three kernels:
//   meta_validate  one block: checks cu_seqlens_q/k, longest key range -> header[5]
//   meta_tokens    one warp per query row: batch, key range, cost
//   meta_split     one block: header fields, prefix sum of costs, per-worker ranges
#include "slikl_common.cuh"

namespace slikl {
namespace {

__global__ void meta_validate(Params P) {
    __shared__ int bad_q, bad_k, maxk;
    if (threadIdx.x == 0) { bad_q = 0; bad_k = 0; maxk = 0; }
    __syncthreads();
    for (int64_t b = threadIdx.x; b < P.B; b += blockDim.x) {
        if (P.layout_q == SLIKL_TND) {
            int32_t a = P.cu_q[b], e = P.cu_q[b + 1];
            if (a < 0 || e < a || e > P.T1) bad_q = 1;
            if (b == 0 && a != 0) bad_q = 1;
            if (b == P.B - 1 && e != P.T1) bad_q = 1;
        }
        int32_t len;
        if (P.layout_k == SLIKL_TND) {
            int32_t a = P.cu_k[b], e = P.cu_k[b + 1];
            if (a < 0 || e < a || e > P.T2) bad_k = 1;
            if (b == 0 && a != 0) bad_k = 1;
            if (b == P.B - 1 && e != P.T2) bad_k = 1;
            len = e - a;
        } else {
            len = (int32_t)P.S2;
        }
        atomicMax(&maxk, len);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (bad_q) set_status(P.status, SLIKL_DEV_BAD_CU_SEQLENS_Q);
        if (bad_k) set_status(P.status, SLIKL_DEV_BAD_CU_SEQLENS_K);
        P.status[1] = bad_k ? 1u : 0u;
        P.meta[5] = bad_k ? 0 : maxk;
    }
}

// Batch of query row t: BSND t / S1; TND the last b with cu_seqlens_q[b] <= t.
__device__ int64_t batch_of_row(const Params &P, int64_t t) {
    if (P.layout_q == SLIKL_BSND) return t / P.S1;
    int64_t lo = 0, hi = P.B - 1;     // invariant: answer in [lo, hi]
    while (lo < hi) {
        int64_t mid = (lo + hi + 1) >> 1;
        if (P.cu_q[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void meta_tokens(Params P) {
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= P.T1) return;
    int64_t b = batch_of_row(P, t);
    int32_t kbase, klen;
    if (P.status[1]) { kbase = 0; klen = 0; }
    else if (P.layout_k == SLIKL_BSND) { kbase = (int32_t)(b * P.S2); klen = (int32_t)P.S2; }
    else { kbase = P.cu_k[b]; klen = P.cu_k[b + 1] - kbase; }
    // cost = 1 + number of 128-slot tiles holding an index >= 0
    const int32_t *row = P.idx + t * (int64_t)P.K;
    int tiles = 0;
    uint64_t mask = 0;
    for (int j0 = 0, i = 0; j0 < P.K; j0 += kSlotTile, ++i) {
        bool any = false;
        for (int j = j0 + lane; j < j0 + kSlotTile && j < P.K; j += 32) any |= row[j] >= 0;
        if (__any_sync(0xffffffffu, any)) {
            tiles += 1;
            mask |= uint64_t(1) << i;
        }
    }
    if (lane == 0) {
        P.tok_kbase[t] = kbase;
        P.tok_klen[t] = klen;
        P.tok_cost[t] = 1 + tiles;
        P.tok_tiles[t] = klen > 0 ? mask : 0;
    }
}

__global__ void meta_split(Params P, int workers, int mode) {
    __shared__ int64_t part[1024];
    const int tid = threadIdx.x, nt = blockDim.x;
    const int64_t T1 = P.T1;
    int32_t *meta = P.meta;
    if (tid == 0) {
        int64_t former = T1 > 0 ? (T1 + workers - 1) / workers : 0;
        int64_t remain = former > 0 ? former - 1 : 0;
        int64_t used = T1 < workers ? T1 : workers;
        int64_t former_cores = T1 - used * remain;
        meta[0] = (int32_t)T1;
        meta[1] = (int32_t)former;
        meta[2] = (int32_t)remain;
        meta[3] = (int32_t)(used - former_cores);
        meta[4] = (int32_t)used;
        meta[6] = mode;
        meta[7] = workers;
    }
    if (mode == 0) {
        int64_t former = T1 > 0 ? (T1 + workers - 1) / workers : 0;
        int64_t remain = former > 0 ? former - 1 : 0;
        int64_t used = T1 < workers ? T1 : workers;
        int64_t former_cores = T1 - used * remain;
        for (int c = tid; c < workers; c += nt) {
            int64_t start = c < former_cores ? c * former
                                             : former_cores * former + (c - former_cores) * remain;
            int64_t n = c < former_cores ? former : (c < used ? remain : 0);
            if (c >= used) start = T1;
            meta[kMetaHeader + 2 * c] = (int32_t)start;
            meta[kMetaHeader + 2 * c + 1] = (int32_t)(start + n);
        }
        return;
    }
    // mode 1: exclusive prefix of cost, chunked per thread, then a block scan of chunk sums
    const int64_t chunk = (T1 + nt - 1) / nt;
    const int64_t lo = tid * chunk, hi = lo + chunk < T1 ? lo + chunk : T1;
    int64_t s = 0;
    for (int64_t t = lo; t < hi; ++t) s += P.tok_cost[t];
    part[tid] = s;
    __syncthreads();
    if (tid == 0) {                     // serial scan of nt partial sums (fixed order)
        int64_t run = 0;
        for (int i = 0; i < nt; ++i) { int64_t v = part[i]; part[i] = run; run += v; }
    }
    __syncthreads();
    int64_t run = part[tid];
    for (int64_t t = lo; t < hi; ++t) { P.cost_prefix[t] = run; run += P.tok_cost[t]; }
    if (hi == T1 && lo <= hi) P.cost_prefix[T1] = run;   // the thread whose chunk ends at T1
    if (T1 == 0 && tid == 0) P.cost_prefix[0] = 0;
    __syncthreads();
    __threadfence_block();
    const int64_t C = P.cost_prefix[T1];
    // worker c starts at the first row t with prefix(t) * workers >= c * C
    for (int c = tid; c <= workers; c += nt) {
        int64_t target = (int64_t)c * C;
        int64_t a = 0, b = T1;          // answer in [a, b]; prefix(T1) * workers >= target
        while (a < b) {
            int64_t mid = (a + b) >> 1;
            if (P.cost_prefix[mid] * workers >= target) b = mid; else a = mid + 1;
        }
        if (c < workers) meta[kMetaHeader + 2 * c] = (int32_t)a;
        if (c > 0) meta[kMetaHeader + 2 * c - 1] = (int32_t)a;
    }
}

}  // namespace

cudaError_t launch_metadata(const Params &P, int workers, int mode, cudaStream_t s) {
    meta_validate<<<1, 256, 0, s>>>(P);
    if (P.T1 > 0) {
        int64_t warps = P.T1;
        int64_t blocks = (warps * 32 + 255) / 256;
        meta_tokens<<<(unsigned)blocks, 256, 0, s>>>(P);
    }
    meta_split<<<1, 1024, 0, s>>>(P, workers, mode);
    return cudaGetLastError();
}

}  // namespace slikl
