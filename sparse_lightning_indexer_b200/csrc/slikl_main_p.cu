// Target distribution of the older fused variant, formed on the sm_100a tensor cores.
//
// aclnnSparseLightningIndexerKLLossGrad (sections "功能说明" and "计算公式") describes the older
// SparseLightningIndexerGradKLLoss as computing the target distribution p inside its kernel
// from the main attention's scores, summed over the heads and L1-normalised. The reading
// taken here: for query row t and main-attention head h,
//
//   A_h(t, j) = softmax over the row's valid slots j of  scale * q_m[t, h] . k_m[key(t, j)]
//   p(t, j)   = (sum_h A_h(t, j)) / (sum_j sum_h A_h(t, j)) = (1 / Nm) sum_h A_h(t, j)
//
// (each head's softmax sums to one over the same slots, so the L1 norm of the head sum is
// Nm). Invalid slots and rows without a valid slot get p = 0.
//
// Per CTA, the query rows of its range from the work split, and for each row two passes over
// its non-empty 128-slot tiles (pass 1: each head's running max and sum; pass 2: the
// normalised weights, summed over the heads):
//   S [128 heads x 128 slots] = q_m[t] . K_m^T   (tcgen05, M = 128 heads, N = 128 slots,
//                                                  K = Dm; fp32 in TMEM, two buffers)
// Heads sit on the TMEM lanes, so a head's max and sum over the slots stay in one thread.
// In pass 2 each head writes its weights into an fp32 [heads x slots] tile in shared memory
// and each slot sums its column over the heads in a fixed order.
//
// Warp roles (384 threads):
//   warps 0-2   producers: the key rows of every tile gathered with cp.async (16-byte chunks,
//               zero-fill for invalid slots); warp 0 also loads q_m[t] by TMA (heads past Nm
//               read as zero) and writes the tile's valid-slot mask into a 4-entry ring
//   warp 3      MMA issuer (one thread) and TMEM owner
//   warps 4-11  softmax groups: thread = head (pass 1 and 2; warps 4-7 take the slot columns
//               0-63, warps 8-11 the columns 64-127, two warps per TMEM lane quadrant so
//               that the exponentials of a sub-partition come from two instruction streams),
//               then thread = slot (column sums)
// Every mbarrier wait is bounded (about one second of SM clock); on expiry the CTA sets
// SLIKL_DEV_WAIT_TIMEOUT, every role stops, in-flight copies and MMAs are drained, TMEM is
// freed and the kernel returns.
#include <type_traits>

#include "slikl_sm100.cuh"

namespace slikl {
namespace {

using namespace sm100;

constexpr int kMpThreads = 384;
constexpr int kMpStages = 2;             // key-row stages of 128 rows x 256 B
constexpr int kMpTmemCols = 256;         // two S buffers [128 heads x 128 slots]
constexpr int kMpStageBytes = 128 * 256;
constexpr int kEStride = 132;            // floats per head row of the weight tile (16-byte rows)
constexpr int kMaskRing = 4;

struct MpBarriers {
    uint64_t kv_full[kMpStages], kv_empty[kMpStages];   // producers -> MMA -> producers
    uint64_t q_full[2], q_empty[2];                     // q_m tiles: producer 0 -> MMA -> producer 0
    uint64_t s_full[2], s_empty[2];                     // S in TMEM: MMA -> softmax -> MMA
    uint64_t mask_full[kMaskRing];                      // tile masks: producer 0 -> softmax
    uint64_t sm_sync;                                   // the 8 softmax warps
    uint64_t drain;
};

struct MpPlan {
    uint32_t kv, q, e, mask, bar, total;
};

__host__ __device__ constexpr uint32_t mp_align(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ constexpr MpPlan mp_plan() {
    return MpPlan{0u,
                  (uint32_t)(kMpStages * kMpStageBytes),
                  (uint32_t)(kMpStages * kMpStageBytes + 2 * 128 * 256),
                  mp_align((uint32_t)(kMpStages * kMpStageBytes + 2 * 128 * 256 + 128 * kEStride * 4), 16),
                  mp_align((uint32_t)(kMpStages * kMpStageBytes + 2 * 128 * 256 + 128 * kEStride * 4), 16) +
                      kMaskRing * 16,
                  mp_align((uint32_t)(kMpStages * kMpStageBytes + 2 * 128 * 256 + 128 * kEStride * 4), 16) +
                      kMaskRing * 16 + (uint32_t)sizeof(MpBarriers) + 1024u};
}

struct MpArgs {
    const void *km;      // [T2][Dm] main-attention key rows
    float *p;            // [T1][K] output
    float scale;
    int Nm, Dm;
};

struct MpItem {
    int pass;            // 0: max and sum; 1: weights and column sums; -1: none
    int t, tile, ord;
    bool first, last;    // first / last tile of the row in this pass
};

// Every role walks the same sequence: for each row of [t0, t1) with a non-empty tile, pass 0
// over its non-empty tiles in index order, then pass 1 over the same tiles.
struct MpSched {
    const uint64_t *tiles;
    int t, t1, ord, pass;
    uint64_t all, m;
    bool first;

    __device__ void advance() {
        for (++t; t < t1; ++t) {
            all = tiles[t];
            if (all) { m = all; pass = 0; first = true; ++ord; return; }
        }
    }
    __device__ void init(const uint64_t *tl, int a, int b) {
        tiles = tl; t = a - 1; t1 = b; ord = -1;
        advance();
    }
    __device__ MpItem next() {
        MpItem it;
        it.pass = -1;
        if (t >= t1) return it;
        it.pass = pass; it.t = t; it.ord = ord; it.first = first;
        it.tile = __ffsll((long long)m) - 1;
        m &= m - 1;
        it.last = m == 0;
        first = false;
        if (it.last) {
            if (pass == 0) { pass = 1; m = all; first = true; }
            else advance();
        }
        return it;
    }
};

template <int Dm, typename T>
__global__ void __launch_bounds__(kMpThreads, 1)
    main_p_sm100(Params P, MpArgs A, const __grid_constant__ CUtensorMap qmap) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr MpPlan SP = mp_plan();
    MpBarriers *bars = reinterpret_cast<MpBarriers *>(smem + SP.bar);
    uint32_t *mask_ring = reinterpret_cast<uint32_t *>(smem + SP.mask);   // [kMaskRing][4]
    __shared__ volatile int abort_flag;
    __shared__ uint32_t tmem_base;
    constexpr int kFmt = std::is_same<T, __nv_bfloat16>::value ? 1 : 0;
    constexpr uint32_t kIdesc = idesc_f16(kFmt, 128, 128, 0, 0);   // both operands K-major
    constexpr int kDChunks = Dm / 8;                               // 16-byte chunks per key row
    constexpr int kRowsPerPass = 32 / kDChunks;                    // 2 (Dm = 128) or 4 (Dm = 64)
    constexpr int kProd = 3;
    const int K = P.K;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = P.meta[kMetaHeader + 2 * blockIdx.x];
    const int t1 = P.meta[kMetaHeader + 2 * blockIdx.x + 1];

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < kMpStages; ++s) {
            mbar_init(&bars->kv_full[s], 32 * kProd);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->q_full[b], 1);
            mbar_init(&bars->q_empty[b], 1);
            mbar_init(&bars->s_full[b], 1);
            mbar_init(&bars->s_empty[b], 8);
        }
        for (int r = 0; r < kMaskRing; ++r) mbar_init(&bars->mask_full[r], 1);
        mbar_init(&bars->sm_sync, 8);
        mbar_init(&bars->drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 3) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&tmem_base)), "r"(kMpTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm_s = tmem_base;

    MpSched sc;
    sc.init(P.tok_tiles, t0, t1);

    if (warp < 3) {
        // =============================== producers ===============================
        const int rsub = lane / kDChunks, chunk = lane % kDChunks;
        const char *kbase_ptr = static_cast<const char *>(A.km);
        int q_last = -1;
        bool ok = true;
        uint32_t g = 0;
        for (MpItem it = sc.next(); ok && it.pass >= 0; it = sc.next(), ++g) {
            if (warp == 0 && it.pass == 0 && it.first) {
                const int qb = it.ord & 1;
                if (!wait_bar(&bars->q_empty[qb], ((it.ord >> 1) & 1) ^ 1, &abort_flag, P.status)) { ok = false; break; }
                if (lane == 0) {
                    const uint32_t qdst = smem_u32(smem + SP.q + qb * 128 * 256);
                    mbar_arrive_expect_tx(&bars->q_full[qb], (Dm / 64) * 128 * 128);
                    tma_load_3d(qdst, &qmap, 0, 0, it.t, &bars->q_full[qb]);
                    if (Dm == 128) tma_load_3d(qdst + 128 * 128, &qmap, 64, 0, it.t, &bars->q_full[qb]);
                }
                q_last = it.ord;
            }
            const int s = g % kMpStages;
            if (!wait_bar(&bars->kv_empty[s], ((g / kMpStages) & 1) ^ 1, &abort_flag, P.status)) { ok = false; break; }
            const int32_t kb = P.tok_kbase[it.t], kl = P.tok_klen[it.t];
            const int32_t *irow = P.idx + (int64_t)it.t * K + it.tile * 128;
            const int jlim = K - it.tile * 128;            // slots of this tile inside the row
            if (warp == 0) {
                // valid-slot mask of the tile (read by the softmax group; the ring entry of item
                // g is rewritten at item g + 4, after the softmax group has finished item g: the
                // stage wait above needs the S product of item g + 2, which needs S buffer g % 2
                // released by the softmax group at the end of item g)
                uint32_t words[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = lane + 32 * u;
                    const int32_t v = j < jlim ? irow[j] : -1;
                    words[u] = __ballot_sync(0xffffffffu, v >= 0 && v < kl);
                }
                if (lane == 0) {
                    uint32_t *mw = mask_ring + (g % kMaskRing) * 4;
                    mw[0] = words[0]; mw[1] = words[1]; mw[2] = words[2]; mw[3] = words[3];
                    mbar_arrive(&bars->mask_full[g % kMaskRing]);
                }
            }
            const uint32_t dst = smem_u32(smem + SP.kv + s * kMpStageBytes) + (chunk >> 3) * 16384;
            // this warp's row groups i = warp, warp + 3, ...: every slot index into registers
            // first (one load latency per tile), then the copies back to back
            constexpr int kGroups = 128 / kRowsPerPass;
            constexpr int kPer = (kGroups + kProd - 1) / kProd;
            int32_t vv[kPer];
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int i = warp + kProd * j;
                const int r = rsub + kRowsPerPass * i;
                vv[j] = (i < kGroups && r < jlim) ? irow[r] : -1;
            }
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int i = warp + kProd * j;
                if (i < kGroups) {
                    const int r = rsub + kRowsPerPass * i;
                    const int32_t v = vv[j];
                    const bool valid = v >= 0 && v < kl;
                    const char *src = kbase_ptr + (valid ? ((int64_t)(kb + v) * (Dm * 2) + chunk * 16) : 0);
                    cp_async16(dst + sw128(r, (chunk & 7) * 8), src, valid ? 16 : 0);
                }
            }
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&bars->kv_full[s]))
                         : "memory");
        }
        cp_async_wait<0>();
        if (!ok && q_last >= 0 && lane == 0) {
            const long long st = clock64();
            while (!mbar_try_wait(&bars->q_full[q_last & 1], (q_last >> 1) & 1) &&
                   clock64() - st < kWaitCycles) {}
        }
    } else if (warp == 3) {
        // =============================== MMA issuer ===============================
        const uint32_t kv0 = smem_u32(smem + SP.kv), q0 = smem_u32(smem + SP.q);
        uint32_t g = 0;
        for (MpItem it = sc.next(); it.pass >= 0; it = sc.next(), ++g) {
            const int s = g % kMpStages, b = g & 1, qb = it.ord & 1;
            if (it.pass == 0 && it.first &&
                !wait_bar(&bars->q_full[qb], (it.ord >> 1) & 1, &abort_flag, P.status)) break;
            if (!wait_bar(&bars->kv_full[s], (g / kMpStages) & 1, &abort_flag, P.status)) break;
            if (!wait_bar(&bars->s_empty[b], ((g >> 1) & 1) ^ 1, &abort_flag, P.status)) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t qaddr = q0 + qb * 128 * 256, kaddr = kv0 + s * kMpStageBytes;
#pragma unroll
                for (int ks = 0; ks < Dm / 16; ++ks) {
                    const uint64_t a = sdesc(qaddr + (ks >> 2) * (128 * 128) + (ks & 3) * 32, 16, 1024);
                    const uint64_t bd = sdesc(kaddr + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                    umma_f16(tm_s + b * 128, a, bd, kIdesc, ks > 0 ? 1u : 0u);
                }
                umma_commit(&bars->s_full[b]);
                umma_commit(&bars->kv_empty[s]);
                if (it.pass == 1 && it.last) umma_commit(&bars->q_empty[qb]);
            }
            __syncwarp();
        }
        if (lane == 0) umma_commit(&bars->drain);
        __syncwarp();
        const long long st = clock64();
        while (!mbar_try_wait(&bars->drain, 0) && clock64() - st < kWaitCycles) {}
    } else {
        // =============================== softmax groups ===============================
        // warps 4-7 take the slot columns 0-63 of every tile, warps 8-11 the columns 64-127;
        // thread = head (lane quadrant warp % 4) in passes 1 and 2, then thread = slot for
        // the column sums (threads 0-127 of the 256)
        const int sw = warp - 4;                     // softmax warp 0..7
        const int half = sw >> 2;                    // column half of the tile
        const int quad = warp & 3;
        const int h = quad * 32 + lane;              // head
        const int et = threadIdx.x - 128;            // 0..255: slot in the sums when < 128
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        float *E = reinterpret_cast<float *>(smem + SP.e);
        const float inv_nm = 1.f / (float)A.Nm;
        __shared__ float st_m[2][128], st_z[2][128];   // per column half: head max and sum
        uint32_t ph = 0, g = 0;
        bool ok = true;
        // rows of the range without a non-empty tile: p = 0
        for (int t = t0; t < t1; ++t) {
            if (P.tok_tiles[t]) continue;
            for (int j = et; j < K; j += 256) A.p[(int64_t)t * K + j] = 0.f;
        }
        float m = -INFINITY, z = 0.f, iz = 0.f;
        for (MpItem it = sc.next(); ok && it.pass >= 0; it = sc.next(), ++g) {
            const int b = g & 1;
            if (!wait_bar(&bars->mask_full[g % kMaskRing], (g / kMaskRing) & 1, &abort_flag, P.status)) { ok = false; break; }
            const uint32_t *mw = mask_ring + (g % kMaskRing) * 4 + 2 * half;
            const uint32_t w0 = mw[0], w1 = mw[1];   // valid-slot bits of this half's two chunks
            if (!wait_bar(&bars->s_full[b], (g >> 1) & 1, &abort_flag, P.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = tm_s + b * 128 + 64 * half + lane_addr;
            if (it.pass == 0) {
                if (it.first) { m = -INFINITY; z = 0.f; }
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    float v[32];
                    tmem_ld32(sa + 32 * c, v);
                    tmem_wait_ld();
                    const uint32_t bits = c == 0 ? w0 : w1;
                    float cm = -INFINITY;
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if ((bits >> k) & 1u) cm = fmaxf(cm, A.scale * v[k]);
                    if (cm > m) {
                        z = (m == -INFINITY) ? 0.f : z * __expf(m - cm);
                        m = cm;
                    }
                    float zs = 0.f;
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if ((bits >> k) & 1u) zs += __expf(A.scale * v[k] - m);
                    z += zs;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->s_empty[b]);
                if (it.last) {
                    // the head's max and sum: this half's, then combined with the other half's
                    // (half 0 first) once every warp has written its own
                    st_m[half][h] = m;
                    st_z[half][h] = z;
                    if (!group_sync(&bars->sm_sync, ph, &abort_flag, P.status)) { ok = false; break; }
                    const float m0 = st_m[0][h], m1 = st_m[1][h];
                    const float M = fmaxf(m0, m1);
                    const float Z = (m0 == -INFINITY ? 0.f : st_z[0][h] * __expf(m0 - M)) +
                                    (m1 == -INFINITY ? 0.f : st_z[1][h] * __expf(m1 - M));
                    m = M;
                    iz = Z > 0.f ? 1.f / Z : 0.f;
                    // st_m / st_z are rewritten at the next row's pass-1 end, after that row's
                    // pass-2 group syncs, which every warp reaches only after these reads
                }
            } else {
                // weights of head h into row h of the tile, this half's 64 columns (heads past
                // Nm are never summed); 16-byte stores, four wavefronts each
                float4 *erow = reinterpret_cast<float4 *>(E + h * kEStride + 64 * half);
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    float v[32];
                    tmem_ld32(sa + 32 * c, v);
                    tmem_wait_ld();
                    const uint32_t bits = c == 0 ? w0 : w1;
                    float e[32];
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        e[k] = ((bits >> k) & 1u) ? __expf(A.scale * v[k] - m) * iz : 0.f;
#pragma unroll
                    for (int k = 0; k < 32; k += 4)
                        erow[(32 * c + k) >> 2] = make_float4(e[k], e[k + 1], e[k + 2], e[k + 3]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->s_empty[b]);
                if (!group_sync(&bars->sm_sync, ph, &abort_flag, P.status)) { ok = false; break; }
                if (et < 128) {
                    // slot et of the tile: its weights summed over the heads in a fixed order
                    // (eight interleaved partial sums, combined pairwise), so the loads overlap
                    float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    int hh = 0;
                    for (; hh + 8 <= A.Nm; hh += 8) {
#pragma unroll
                        for (int u = 0; u < 8; ++u) a8[u] += E[(hh + u) * kEStride + et];
                    }
#pragma unroll
                    for (int u = 0; u < 7; ++u)               // the last Nm % 8 heads
                        if (hh + u < A.Nm) a8[u] += E[(hh + u) * kEStride + et];
                    const float acc = ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
                    const int j = it.tile * 128 + et;
                    if (j < K) A.p[(int64_t)it.t * K + j] = acc * inv_nm;
                }
                if (!group_sync(&bars->sm_sync, ph, &abort_flag, P.status)) { ok = false; break; }
                if (it.last && et < 128) {
                    // p = 0 on the row's empty tiles
                    const uint64_t all = P.tok_tiles[it.t];
                    for (int tl = 0; tl * 128 < K; ++tl) {
                        if ((all >> tl) & 1) continue;
                        const int jz = tl * 128 + et;
                        if (jz < K) A.p[(int64_t)it.t * K + jz] = 0.f;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 3) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm_s),
                     "r"(kMpTmemCols));
    }
}

template <int Dm, typename T>
cudaError_t launch_mp_t(const Params &P, const MpArgs &A, const void *qm, int workers,
                        cudaStream_t s) {
    constexpr MpPlan sp = mp_plan();
    static_assert(sp.total <= 227 * 1024, "main-attention p kernel shared memory");
    // q_m viewed as the indexer's q with Nm heads of Dm: boxes of 64 d x 128 heads x 1 row
    Params Pq = P;
    Pq.q = qm;
    Pq.N1 = A.Nm;
    Pq.D = Dm;
    CUtensorMap qmap;
    cudaError_t e = encode_q_map<128, T>(Pq, &qmap);
    if (e != cudaSuccess) return e;
    auto k = main_p_sm100<Dm, T>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total);
    if (e != cudaSuccess) return e;
    k<<<workers, kMpThreads, sp.total, s>>>(P, A, qmap);
    return cudaGetLastError();
}

}  // namespace

// Shapes: Nm in [1, 128], Dm in {64, 128}; the work split of P (meta) gives each CTA its rows.
cudaError_t launch_main_p(const Params &P, const void *q_main, const void *k_main, float *p_out,
                          float scale, int Nm, int Dm, int workers, cudaStream_t s) {
    if (Nm < 1 || Nm > 128 || (Dm != 64 && Dm != 128)) return cudaErrorInvalidValue;
    if (P.T1 <= 0) return cudaSuccess;
    MpArgs A{k_main, p_out, scale, Nm, Dm};
    if (P.dtype == SLIKL_BF16)
        return Dm == 128 ? launch_mp_t<128, __nv_bfloat16>(P, A, q_main, workers, s)
                         : launch_mp_t<64, __nv_bfloat16>(P, A, q_main, workers, s);
    return Dm == 128 ? launch_mp_t<128, __half>(P, A, q_main, workers, s)
                     : launch_mp_t<64, __half>(P, A, q_main, workers, s);
}

}  // namespace slikl
