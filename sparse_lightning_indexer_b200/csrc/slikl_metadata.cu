// Work split ("metadata") of the merged B*S1 query rows over the CTAs of the fused kernel.
//
// The analogue of the DenseLightningIndexerKLLossGradMetadata AICPU operator (article on
// that operator, sections "功能定位" and "Metadata 输出布局"): there the merged rows are cut
// into formerCoreSize = ceil(total / cores) and remainCoreSize = formerCoreSize - 1 pieces.
// Here the split runs on the device, next to the data, and can also balance a per-row cost
// (mode 1) because the cost of a query row grows with its number of non-empty slot tiles.
//
// Three kernels:
//   meta_validate  one block: checks cu_seqlens_q/k, longest key range -> header[5]; for the
//                  key-major dK path also the first unit of every batch
//   meta_tokens    one warp per query row: batch, key range in use, index-contract check,
//                  cost, non-empty slot tiles and (key-major path) the 256-key block pairs
//                  the row names
//   meta_split     one block: header fields, prefix sum of costs, per-worker ranges
// and two for the key-major dK path:
//   km_units       one warp per unit (32 query rows of a batch x one 256-key block pair):
//                  which of the 32 rows name a key of the pair
//   km_split       one block: drops the empty units, then cost-balanced contiguous ranges of
//                  the rest, one per worker
#include "slikl_common.cuh"

namespace slikl {
namespace {

// Exclusive prefix sum of get(0..n-1) into out[0..n] (out[n] = total) by one block of up to
// 1024 threads: contiguous chunks per thread, a block scan of the chunk sums, and a second
// pass over each chunk. The summation order is fixed.
template <typename F>
__device__ void block_prefix(int64_t n, F get, int64_t *out) {
    __shared__ int64_t warp_tot[32];
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, wid = tid >> 5;
    const int64_t chunk = (n + nt - 1) / nt;
    const int64_t lo = (int64_t)tid * chunk < n ? (int64_t)tid * chunk : n;
    const int64_t hi = lo + chunk < n ? lo + chunk : n;
    int64_t s = 0;
    for (int64_t i = lo; i < hi; ++i) s += get(i);
    int64_t x = s;                                  // inclusive scan within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
        const int nw = (nt + 31) >> 5;
        int64_t w = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < nw) warp_tot[lane] = w;         // inclusive over warps
    }
    __syncthreads();
    int64_t run = x - s + (wid > 0 ? warp_tot[wid - 1] : 0);
    for (int64_t i = lo; i < hi; ++i) { out[i] = run; run += get(i); }
    if (tid == nt - 1) out[n] = warp_tot[(nt - 1) >> 5];
    __syncthreads();
}

// Query rows [q0, q1) and key rows [k0, k0 + klen) of batch b (klen = 0 when cu_seqlens_k
// is unusable).
__device__ void batch_ranges(const Params &P, int64_t b, int64_t &q0, int64_t &q1, int64_t &k0,
                             int64_t &klen) {
    if (P.layout_q == SLIKL_BSND) { q0 = b * P.S1; q1 = q0 + P.S1; }
    else { q0 = P.cu_q[b]; q1 = P.cu_q[b + 1]; }
    if (P.status[1]) { k0 = 0; klen = 0; }
    else if (P.layout_k == SLIKL_BSND) { k0 = b * P.S2; klen = P.S2; }
    else { k0 = P.cu_k[b]; klen = P.cu_k[b + 1] - k0; }
}

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
        if (P.km && !bad_k && maxk > P.kbound) set_status(P.status, SLIKL_DEV_KEY_RANGE_ABOVE_S2);
        P.status[1] = bad_k ? 1u : 0u;
        P.meta[5] = bad_k ? 0 : maxk;
    }
    __syncthreads();
    if (P.km) {
        // units of batch b: ceil(query rows / 32) x ceil(key rows / 256); none when the
        // batch's ranges are unusable or longer than the record rows
        const bool none = bad_q || bad_k;
        block_prefix(
            P.B,
            [&](int64_t b) -> int64_t {
                if (none) return 0;
                int64_t q0, q1, k0, klen;
                batch_ranges(P, b, q0, q1, k0, klen);
                if (klen > P.S2m || q1 <= q0 || klen <= 0) return 0;
                return ((q1 - q0 + 31) / 32) * ((klen + 255) / 256);
            },
            P.unit_off);
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
    const int64_t b = batch_of_row(P, t);
    int64_t q0, q1, k0, kfull;
    batch_ranges(P, b, q0, q1, k0, kfull);
    // rows and keys of the batch in use (seqUsedQ / seqUsedK), clamped into its ranges
    bool in_use = true;
    int64_t kuse = kfull;
    if (P.used_q) {
        const int64_t u = P.used_q[b], n = q1 - q0 > 0 ? q1 - q0 : 0;
        const int64_t c = u < 0 ? 0 : (u > n ? n : u);
        if (c != u && lane == 0) set_status(P.status, SLIKL_DEV_BAD_SEQ_USED);
        in_use = t - q0 < c;
    }
    if (P.used_k) {
        const int64_t u = P.used_k[b];
        const int64_t c = u < 0 ? 0 : (u > kfull ? kfull : u);
        if (c != u && lane == 0) set_status(P.status, SLIKL_DEV_BAD_SEQ_USED);
        kuse = c;
    }
    const int32_t kbase = (int32_t)k0;
    const int32_t klen = in_use ? (int32_t)kuse : 0;   // a slot is valid when 0 <= v < klen
    // cost = 1 + number of 128-slot tiles holding a valid index; lane l reads slots
    // 4l..4l+3 of each tile (one 16-byte load when the row is 16-byte aligned). Every index
    // of a row in use is checked against the batch's whole key range (a padding row's
    // indices are not read).
    const int32_t *row = P.idx + t * (int64_t)P.K;
    const bool vec = (P.K & 3) == 0;
    const bool check = !P.status[1];
    const int32_t klim = P.km ? (klen < P.S2m ? klen : P.S2m) : 0;
    int tiles = 0;
    uint64_t mask = 0;
    uint32_t pw0 = 0, pw1 = 0;           // 256-key block pairs named (key-major path, <= 64)
    bool bad = false;
    const int ntiles = in_use ? (P.K + kSlotTile - 1) / kSlotTile : 0;
#pragma unroll 4
    for (int i = 0; i < ntiles; ++i) {
        const int j = i * kSlotTile + 4 * lane;
        int v[4] = {-1, -1, -1, -1};
        if (vec) {
            if (j < P.K) {
                const int4 x = *reinterpret_cast<const int4 *>(row + j);
                v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
            }
        } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = j + u < P.K ? row[j + u] : -1;
        }
        bool any = false;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            bad |= check && (v[u] < -1 || v[u] >= kfull);
            any |= v[u] >= 0 && v[u] < klen;
            if (v[u] >= 0 && v[u] < klim) {
                const int kp = v[u] >> 8;
                const uint32_t bit = 1u << (kp & 31);
                if (kp < 32) pw0 |= bit; else pw1 |= bit;
            }
        }
        if (__any_sync(0xffffffffu, any)) {
            tiles += 1;
            mask |= uint64_t(1) << i;
        }
    }
    if (bad) set_status(P.status, SLIKL_DEV_INDEX_OUT_OF_RANGE);
    if (P.km) {
        pw0 = __reduce_or_sync(0xffffffffu, pw0);
        pw1 = __reduce_or_sync(0xffffffffu, pw1);
        if (lane < P.nkpw) P.tok_pairs[t * P.nkpw + lane] = lane == 0 ? pw0 : pw1;
    }
    if (lane == 0) {
        P.tok_kbase[t] = kbase;
        P.tok_klen[t] = klen;
        P.tok_cost[t] = 1 + tiles;
        P.tok_tiles[t] = klen > 0 ? mask : 0;
    }
}

__global__ void meta_split(Params P, int workers, int mode) {
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
    // mode 1: exclusive prefix of cost
    block_prefix(T1, [&](int64_t t) -> int64_t { return P.tok_cost[t]; }, P.cost_prefix);
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

// One warp per candidate unit u < units_max; units past the count are left alone.
__global__ void km_units(Params P) {
    const int lane = threadIdx.x & 31;
    const int64_t u = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t total = P.unit_off[P.B];
    if (u >= total) return;
    int64_t lo = 0, hi = P.B - 1;        // last batch with unit_off[b] <= u
    while (lo < hi) {
        const int64_t mid = (lo + hi + 1) >> 1;
        if (P.unit_off[mid] <= u) lo = mid; else hi = mid - 1;
    }
    const int64_t b = lo;
    int64_t q0, q1, k0, klen;
    batch_ranges(P, b, q0, q1, k0, klen);
    const int64_t nch = (q1 - q0 + 31) / 32;
    const int64_t r = u - P.unit_off[b];
    const int kp = (int)(r / nch);
    const int64_t tok0 = q0 + (r % nch) * 32;
    const int64_t t = tok0 + lane;
    bool on = false;
    if (t < q1) on = (P.tok_pairs[t * P.nkpw + (kp >> 5)] >> (kp & 31)) & 1u;
    const uint32_t m = __ballot_sync(0xffffffffu, on);
    if (lane == 0) {
        const int64_t rest = klen - 256 * (int64_t)kp;
        const int nkeys = rest < 256 ? (int)rest : 256;
        P.units[u] = make_int4((int)tok0, (int)(k0 + 256 * kp), (256 * kp) | (nkeys << 16), (int)m);
    }
}

__global__ void km_split(Params P, int workers) {
    const int64_t n_all = P.unit_off[P.B];
    // keep the units that hold at least one row (their order is kept)
    block_prefix(n_all, [&](int64_t u) -> int64_t { return P.units[u].w != 0 ? 1 : 0; },
                 P.unit_prefix);
    __threadfence_block();
    for (int64_t u = threadIdx.x; u < n_all; u += blockDim.x) {
        const int4 x = P.units[u];
        if (x.w != 0) P.units_c[P.unit_prefix[u]] = x;
    }
    const int64_t n = P.unit_prefix[n_all];
    __syncthreads();
    __threadfence_block();
    // cost of a unit: a small fixed part plus its row count
    block_prefix(n, [&](int64_t u) -> int64_t { return 1 + 8 * __popc((uint32_t)P.units_c[u].w); },
                 P.unit_prefix);
    __threadfence_block();
    const int64_t C = P.unit_prefix[n];
    for (int c = threadIdx.x; c <= workers; c += blockDim.x) {
        const int64_t target = (int64_t)c * C;
        int64_t a = 0, bb = n;           // first unit with prefix * workers >= target
        while (a < bb) {
            const int64_t mid = (a + bb) >> 1;
            if (P.unit_prefix[mid] * workers >= target) bb = mid; else a = mid + 1;
        }
        P.km_range[c] = (int32_t)(c == workers ? n : a);
    }
}

}  // namespace

cudaError_t launch_km_metadata(const Params &P, int workers, cudaStream_t s) {
    if (P.units_max > 0) {
        const int64_t blocks = (P.units_max * 32 + 255) / 256;
        km_units<<<(unsigned)blocks, 256, 0, s>>>(P);
    }
    km_split<<<1, 1024, 0, s>>>(P, workers);
    return cudaGetLastError();
}

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
