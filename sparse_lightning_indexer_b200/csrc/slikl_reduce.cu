// dK finishing kernels.
//
// Atomic mode (the page's default, "确定性计算": non-deterministic), and deterministic mode on
// the key-major path: fp32 dK rows are in dk_acc; cast_dk converts them to the input dtype.
//
// Deterministic mode on the scatter path: the fused kernel stored one fp32 dK row per slot (t, j) in
// `partials`. The slots are then inverted into key-major order by a stable LSD radix sort
// on (key row, slot id) — hand-written, 8-bit digits — giving a CSR over key rows, and every
// key row sums its slots in ascending slot-id order, so the result is bitwise reproducible.
#include "slikl_common.cuh"

namespace slikl {
namespace {

__global__ void cast_dk(const float *__restrict__ acc, void *dk, int64_t n4, int dtype) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x) {
        float4 v = reinterpret_cast<const float4 *>(acc)[i];
        if (dtype == SLIKL_BF16) {
            __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
            uint2 o;
            o.x = *reinterpret_cast<uint32_t *>(&a);
            o.y = *reinterpret_cast<uint32_t *>(&b);
            reinterpret_cast<uint2 *>(dk)[i] = o;
        } else {
            __half2 a = __floats2half2_rn(v.x, v.y), b = __floats2half2_rn(v.z, v.w);
            uint2 o;
            o.x = *reinterpret_cast<uint32_t *>(&a);
            o.y = *reinterpret_cast<uint32_t *>(&b);
            reinterpret_cast<uint2 *>(dk)[i] = o;
        }
    }
}

// keys = key row of slot i (T2 for an invalid slot), vals = slot id i = t*K + j
__global__ void sort_init(Params P, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        int64_t t = i / P.K;
        int32_t r = slot_row(P.idx[i], P.tok_kbase[t], P.tok_klen[t]);
        P.keys0[i] = r >= 0 ? r : (int32_t)P.T2;
        P.vals0[i] = (int32_t)i;
    }
}

__global__ void sort_hist(const int32_t *__restrict__ keys, int64_t n, int shift, int32_t *hist,
                          int nblocks) {
    __shared__ int cnt[256];
    for (int d = threadIdx.x; d < 256; d += blockDim.x) cnt[d] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kSortTile;
    for (int e = threadIdx.x; e < kSortTile; e += blockDim.x) {
        int64_t i = base + e;
        if (i < n) atomicAdd(&cnt[(keys[i] >> shift) & 255], 1);
    }
    __syncthreads();
    for (int d = threadIdx.x; d < 256; d += blockDim.x) hist[(int64_t)d * nblocks + blockIdx.x] = cnt[d];
}

// Exclusive scan of m ints in place (one block, fixed order).
__global__ void scan_exclusive(int32_t *a, int64_t m) {
    __shared__ int64_t part[1024];
    const int tid = threadIdx.x, nt = blockDim.x;
    const int64_t chunk = (m + nt - 1) / nt;
    const int64_t lo = tid * chunk, hi = lo + chunk < m ? lo + chunk : m;
    int64_t s = 0;
    for (int64_t i = lo; i < hi; ++i) s += a[i];
    part[tid] = s;
    __syncthreads();
    if (tid == 0) {
        int64_t run = 0;
        for (int i = 0; i < nt; ++i) { int64_t v = part[i]; part[i] = run; run += v; }
    }
    __syncthreads();
    int64_t run = part[tid];
    for (int64_t i = lo; i < hi; ++i) { int32_t v = a[i]; a[i] = (int32_t)run; run += v; }
}

// Stable scatter of one radix pass. 8 warps; warp w owns elements [w*512, (w+1)*512) of the
// block's tile and ranks them in order with match_any, so equal digits keep input order.
__global__ void __launch_bounds__(256) sort_scatter(const int32_t *__restrict__ kin,
                                                    const int32_t *__restrict__ vin,
                                                    int32_t *kout, int32_t *vout, int64_t n,
                                                    int shift, const int32_t *hist, int nblocks) {
    __shared__ int wcount[8][257];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < 8 * 257; e += blockDim.x) (&wcount[0][0])[e] = 0;
    __syncthreads();
    const int64_t wbase = (int64_t)blockIdx.x * kSortTile + warp * (kSortTile / 8);
    constexpr int kRounds = kSortTile / 8 / 32;
    for (int r = 0; r < kRounds; ++r) {
        int64_t i = wbase + r * 32 + lane;
        int dg = i < n ? (kin[i] >> shift) & 255 : 256;
        unsigned peers = __match_any_sync(0xffffffffu, dg);
        if (dg < 256 && lane == __ffs(peers) - 1) wcount[warp][dg] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    for (int d = threadIdx.x; d < 256; d += blockDim.x) {
        int run = hist[(int64_t)d * nblocks + blockIdx.x];
        for (int w = 0; w < 8; ++w) { int c = wcount[w][d]; wcount[w][d] = run; run += c; }
    }
    __syncthreads();
    const unsigned lt = (1u << lane) - 1u;
    for (int r = 0; r < kRounds; ++r) {
        int64_t i = wbase + r * 32 + lane;
        int32_t key = i < n ? kin[i] : 0;
        int dg = i < n ? (key >> shift) & 255 : 256;
        unsigned peers = __match_any_sync(0xffffffffu, dg);
        if (dg < 256) {
            int pos = wcount[warp][dg] + __popc(peers & lt);
            kout[pos] = key;
            vout[pos] = vin[i];
        }
        __syncwarp();
        if (dg < 256 && lane == __ffs(peers) - 1) wcount[warp][dg] += __popc(peers);
        __syncwarp();
    }
}

// row_ptr[r] = first sorted position whose key is >= r, for r in [0, T2 + 1].
__global__ void csr_rows(const int32_t *__restrict__ keys, int64_t n, int32_t *row_ptr, int64_t T2) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i <= n;
         i += (int64_t)gridDim.x * blockDim.x) {
        int64_t prev = i == 0 ? -1 : keys[i - 1];
        int64_t cur = i == n ? T2 + 1 : keys[i];
        for (int64_t r = prev + 1; r <= cur; ++r) row_ptr[r] = (int32_t)i;
    }
}

// One warp per key row: sum its slots' partial rows in ascending slot id, cast, store.
__global__ void segmented_reduce(Params P, const int32_t *__restrict__ vals) {
    const int lane = threadIdx.x & 31;
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (r >= P.T2) return;
    const int D = P.D;
    const int per_lane = D / 32;     // 4 (D = 128) or 2 (D = 64)
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int32_t a = P.row_ptr[r], e = P.row_ptr[r + 1];
    for (int32_t s = a; s < e; ++s) {
        const float *src = P.partials + (int64_t)vals[s] * D + lane * per_lane;
        if (per_lane == 4) {
            float4 v = *reinterpret_cast<const float4 *>(src);
            acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
        } else {
            float2 v = *reinterpret_cast<const float2 *>(src);
            acc[0] += v.x; acc[1] += v.y;
        }
    }
    for (int c = 0; c < per_lane; ++c) store_from_float(P.dk, r * D + lane * per_lane + c, acc[c], P.dtype);
}

int grid_for(int64_t n, int threads) {
    int64_t b = (n + threads - 1) / threads;
    if (b > 148 * 32) b = 148 * 32;
    return (int)(b > 0 ? b : 1);
}

}  // namespace

cudaError_t launch_cast(const Params &P, cudaStream_t s) {
    int64_t n4 = P.T2 * (int64_t)P.D / 4;
    if (n4 > 0) cast_dk<<<grid_for(n4, 256), 256, 0, s>>>(P.dk_acc, P.dk, n4, P.dtype);
    return cudaGetLastError();
}

cudaError_t launch_deterministic_reduce(const Params &P, cudaStream_t s) {
    const int64_t n = P.T1 * (int64_t)P.K;
    if (P.T2 == 0) return cudaGetLastError();
    if (n == 0) {
        size_t bytes = (size_t)P.T2 * P.D * (P.dtype == SLIKL_BF16 ? 2 : 2);
        return cudaMemsetAsync(P.dk, 0, bytes, s);
    }
    const int nblocks = (int)((n + kSortTile - 1) / kSortTile);
    sort_init<<<grid_for(n, 256), 256, 0, s>>>(P, n);
    int nbits = 0;
    while ((int64_t(1) << nbits) <= P.T2) ++nbits;          // keys lie in [0, T2]
    const int passes = (nbits + 7) / 8;
    int32_t *kin = P.keys0, *vin = P.vals0, *kout = P.keys1, *vout = P.vals1;
    for (int ps = 0; ps < passes; ++ps) {
        sort_hist<<<nblocks, 256, 0, s>>>(kin, n, 8 * ps, P.hist, nblocks);
        scan_exclusive<<<1, 1024, 0, s>>>(P.hist, (int64_t)256 * nblocks);
        sort_scatter<<<nblocks, 256, 0, s>>>(kin, vin, kout, vout, n, 8 * ps, P.hist, nblocks);
        int32_t *tk = kin, *tv = vin;
        kin = kout; vin = vout; kout = tk; vout = tv;
    }
    csr_rows<<<grid_for(n + 1, 256), 256, 0, s>>>(kin, n, P.row_ptr, P.T2);
    int64_t warps = P.T2;
    segmented_reduce<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, s>>>(P, vin);
    return cudaGetLastError();
}

}  // namespace slikl
