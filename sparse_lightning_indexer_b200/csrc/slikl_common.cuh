// Shared definitions of the CUDA library: problem parameters as the kernels see them,
// the workspace layout, device status bits and small device helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "slikl.h"

namespace slikl {

constexpr int kMaxWorkers = 4096;        // metadata capacity (workers = CTAs of the fused kernel)
constexpr int kKmDetWorkers = 256;       // most CTAs of the key-major kernel in deterministic mode
                                         // (its per-CTA scratch is sized for this many)
constexpr int kSlotTile = 128;           // top-k slots per tile of the fused kernel
constexpr int kMetaHeader = 8;

// Everything a kernel needs about one call. Built on the host, passed by value.
struct Params {
    int dtype;            // SLIKL_FP16 / SLIKL_BF16
    int layout_q, layout_k;
    int deterministic;
    int64_t B, S1, S2;    // BSND lengths (0 when that side is TND)
    int64_t T1, T2;       // total query / key rows
    int N1, D, K;         // heads, head dim, top-k
    const void *q, *k;
    const float *w, *p;
    const int32_t *idx, *cu_q, *cu_k;
    const int32_t *used_q, *used_k;   // [B] rows of each batch in use, or null (all in use)
    void *dq, *dk;
    float *dw, *y;
    // workspace regions
    uint32_t *status;     // device status word(s)
    int32_t *meta;        // [kMetaHeader + 2*workers]
    int32_t *tok_kbase;   // [T1] first key row of the token's batch
    int32_t *tok_klen;    // [T1] keys of the token's batch in use (0 for a padding row); a
                          // slot is valid when 0 <= index < tok_klen
    int32_t *tok_cost;    // [T1] work estimate per token
    uint64_t *tok_tiles;  // [T1] bit i set when slot tile i holds a valid index
    int64_t *cost_prefix; // [T1 + 1]
    float *dk_acc;        // [T2*D] fp32 accumulator (atomic mode)
    float *partials;      // [T1*K*D] per-slot dK rows (deterministic mode)
    int32_t *keys0, *vals0, *keys1, *vals1;   // radix-sort buffers [T1*K]
    int32_t *hist;        // [256 * sort_blocks]
    int32_t *row_ptr;     // [T2 + 2]
    // key-major dK path (km = 1): the fused kernel stores one record per named (token, key)
    // and the key-major kernel forms dK block by block from them
    int km;
    int S2m;              // record row length in keys: longest key range rounded up to 256
    int64_t kbound;       // the longest key range the caller promised
    int nkpw;             // 32-bit words per token in tok_pairs
    int rec_bytes;        // 8 (N1 <= 32; 16 in deterministic mode), 16 (N1 <= 64), 32 (N1 <= 128)
    uint32_t *tok_pairs;  // [T1][nkpw] bit kp: the token names a key of [256 kp, 256 kp + 256)
    void *rec;            // [T1][S2m] records {dI, ReLU(S) > 0 mask of the heads}
    int4 *units;          // [units_max] {first token, first key row, local key | keys << 16,
                          //              token mask}: 32 tokens x one 256-key block pair
    int4 *units_c;        // [units_max] the units that hold at least one row, in order
    int64_t *unit_off;    // [B + 1] first unit of each batch; unit_off[B] = unit count
    int64_t *unit_prefix; // [units_max + 1] exclusive prefix of the unit costs
    int32_t *km_range;    // [kMaxWorkers + 1] first unit of each worker of the key-major kernel
    int64_t units_max;
    // deterministic key-major path: the runs of 256-key block pairs that a CTA's unit range
    // cuts (its first run, continued from the previous CTA, and its last, continued by the
    // next) are stored here instead of added, [kKmDetWorkers][2][256][D], and summed in CTA
    // order afterwards
    float *km_scratch;
    // key-major path: q scaled by the head weights, w_th q_th, [T1][N1][D] in the input type
    void *km_qw;
};

// Shape of the key-major dK path of one call (km = 0: scatter path).
struct KmShape {
    int km;
    int S2m, nkpw, rec_bytes;
    int64_t units_max, kbound;
    int64_t qw_bytes;     // the w-scaled copy of q
};

// Byte offsets of the workspace regions; every region starts 256-byte aligned.
struct WsLayout {
    size_t status, meta, tok_kbase, tok_klen, tok_cost, tok_tiles, cost_prefix;
    size_t dk_acc, partials, keys0, vals0, keys1, vals1, hist, row_ptr;
    size_t tok_pairs, rec, units, units_c, unit_off, unit_prefix, km_range, km_scratch, km_qw;
    size_t total;
};

constexpr int kSortTile = 4096;          // elements per block of one radix-sort pass

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout make_layout(int64_t T1, int64_t T2, int64_t K, int64_t D, int det,
                            const KmShape &km = KmShape{}, int64_t B = 0) {
    WsLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
    L.status = take(256);
    L.meta = take(sizeof(int32_t) * (kMetaHeader + 2 * kMaxWorkers));
    L.tok_kbase = take(sizeof(int32_t) * (size_t)T1);
    L.tok_klen = take(sizeof(int32_t) * (size_t)T1);
    L.tok_cost = take(sizeof(int32_t) * (size_t)T1);
    L.tok_tiles = take(sizeof(uint64_t) * (size_t)T1);
    L.cost_prefix = take(sizeof(int64_t) * (size_t)(T1 + 1));
    const bool k = km.km != 0;
    const bool sorted = det && !k;           // deterministic mode on the scatter path
    L.dk_acc = take(sorted ? 0 : sizeof(float) * (size_t)T2 * (size_t)D);
    size_t n = (size_t)T1 * (size_t)K;
    size_t sort_blocks = (n + kSortTile - 1) / kSortTile;
    L.partials = take(sorted ? sizeof(float) * n * (size_t)D : 0);
    L.keys0 = take(sorted ? sizeof(int32_t) * n : 0);
    L.vals0 = take(sorted ? sizeof(int32_t) * n : 0);
    L.keys1 = take(sorted ? sizeof(int32_t) * n : 0);
    L.vals1 = take(sorted ? sizeof(int32_t) * n : 0);
    L.hist = take(sorted ? sizeof(int32_t) * 256 * sort_blocks : 0);
    L.row_ptr = take(sorted ? sizeof(int32_t) * (size_t)(T2 + 2) : 0);
    L.tok_pairs = take(k ? sizeof(uint32_t) * (size_t)T1 * km.nkpw : 0);
    L.rec = take(k ? (size_t)T1 * (size_t)km.S2m * km.rec_bytes : 0);
    L.units = take(k ? 16 * (size_t)km.units_max : 0);
    L.units_c = take(k ? 16 * (size_t)km.units_max : 0);
    L.unit_off = take(k ? sizeof(int64_t) * (size_t)(B + 1) : 0);
    L.unit_prefix = take(k ? sizeof(int64_t) * (size_t)(km.units_max + 1) : 0);
    L.km_range = take(k ? sizeof(int32_t) * (kMaxWorkers + 1) : 0);
    L.km_scratch = take(k && det ? sizeof(float) * (size_t)kKmDetWorkers * 2 * 256 * (size_t)D : 0);
    L.km_qw = take(k ? (size_t)km.qw_bytes : 0);
    L.total = off;
    return L;
}

// status word layout: status[0] = SLIKL_DEV_* bits; status[1] = 1 when cu_seqlens_k is
// unusable (every batch's key range is then empty); status[2..] reserved.

__device__ __forceinline__ void set_status(uint32_t *status, uint32_t bit) {
    atomicOr(status, bit);
}

__device__ __forceinline__ float load_as_float(const void *base, size_t i, int dtype) {
    if (dtype == SLIKL_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base)[i]);
    return __half2float(reinterpret_cast<const __half *>(base)[i]);
}

__device__ __forceinline__ void store_from_float(void *base, size_t i, float v, int dtype) {
    if (dtype == SLIKL_BF16) reinterpret_cast<__nv_bfloat16 *>(base)[i] = __float2bfloat16_rn(v);
    else reinterpret_cast<__half *>(base)[i] = __float2half_rn(v);
}

__device__ __forceinline__ void red_add_f32(float *addr, float v) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}

// Key-major records: the mask words of the heads, then dI at this byte offset. In
// deterministic mode dI is a signed 64-bit fixed-point number (units of 2^-48) summed with
// integer adds, so repeated slots of a key give the same sum in any order; |dI| <= 1 per slot
// and at most 8192 slots per row keep the sum below 2^61.
__host__ __device__ constexpr int rec_di_offset(int rec_bytes) { return rec_bytes == 8 ? 4 : rec_bytes / 2; }
constexpr float kDiFixedOne = 281474976710656.0f;    // 2^48

__device__ __forceinline__ void red_add_di_fixed(void *addr, float dI) {
    const long long v = __float2ll_rn(dI * kDiFixedOne);
    asm volatile("red.global.add.u64 [%0], %1;" ::"l"(addr), "l"(v) : "memory");
}

__device__ __forceinline__ float di_from_fixed(long long v) {
    return __ll2float_rn(v) * (1.0f / kDiFixedOne);
}

// Key row of slot value v for a token whose keys in use are [kbase, kbase + klen), or -1.
// (Values that break the index contract were flagged by the metadata pass; here they are
// simply invalid.)
__device__ __forceinline__ int32_t slot_row(int32_t v, int32_t kbase, int32_t klen) {
    return v >= 0 && v < klen ? kbase + v : -1;
}

// kernels (defined in the .cu files)
cudaError_t launch_metadata(const Params &P, int workers, int mode, cudaStream_t s);
cudaError_t launch_fused_sm100(const Params &P, int workers, cudaStream_t s);
cudaError_t launch_fused_pair_sm100(const Params &P, int workers, cudaStream_t s);
cudaError_t launch_cast(const Params &P, cudaStream_t s);
cudaError_t launch_deterministic_reduce(const Params &P, cudaStream_t s);
cudaError_t launch_km_metadata(const Params &P, int workers, cudaStream_t s);
cudaError_t launch_dk_keymajor(const Params &P, int workers, cudaStream_t s);
cudaError_t launch_km_det_combine(const Params &P, int workers, cudaStream_t s);
cudaError_t launch_main_p(const Params &P, const void *q_main, const void *k_main, float *p_out,
                          float scale, int Nm, int Dm, int workers, cudaStream_t s);
cudaError_t launch_dense_indices(int32_t *idx, int64_t T1, int64_t B, int64_t S1, int64_t S2,
                                 int Ld, int layout_q, int layout_k, int mask,
                                 const int32_t *cu_q, const int32_t *cu_k, const int32_t *used_q,
                                 const int32_t *used_k, uint32_t *flag, cudaStream_t s);
cudaError_t launch_dense_flag_merge(const uint32_t *flag, uint32_t *status, cudaStream_t s);

}  // namespace slikl
