// Key-major dK on the sm_100a tensor cores (tcgen05 MMA, accumulators in TMEM).
//
// The operator adds dK_topk(t) = dS_t^T . q_t into the key rows named by each query row t
// (aclnnSparseLightningIndexerKLLossGrad, section "计算公式"). Grouped by key instead of by
// query row, the same sum reads
//
//   dK_j = sum over the rows t that name key j of  sum_h dS_t[h, j] q_t[h, :]
//
// The fused kernel leaves one record per named (t, j): dI_tj and the set of heads with
// S_tjh > 0. With dS_tjh = dI_tj * w_th * [S_tjh > 0], the head weight moves to q:
//
//   dK_j = sum_t sum_h (w_th q_th) (dI_tj [S_tjh > 0])
//
// km_scale_q forms qw_th = w_th q_th once per call (fp32 product rounded to the input type),
// the dS builders here form dI_tj [S_tjh > 0] (dI rounded to the input type) from the
// records alone, and for one 256-key block pair the products of all rows that name a key of
// the pair accumulate in TMEM:
//
//   dK^T [D x 256 keys] += qw_t^T [D x heads] . dS'_t [heads x 256 keys]   (M = 128, N = 256)
//
// so a key row takes one fp32 add per run of work units instead of one per naming slot.
//
// Rows of fewer than 64 heads are packed into one stage: G = 64 / N1P query rows of a run
// share the stage's 64-wide contraction (row g's heads are contraction indices g*N1P ..
// g*N1P + N1P - 1), so a stage carries 64 contraction indices whatever N1. The MMAs of a
// stage are issued row after row, as with one row per stage, so the sum order is unchanged.
//
// Work units are 32 query rows of one batch x one 256-key block pair (tables built by the
// key-major metadata kernels). Each CTA takes a contiguous, cost-balanced range of units;
// consecutive units on the same pair form a run that accumulates in one of two TMEM
// buffers and is flushed once, with red.global.add.f32 of 32 consecutive d per warp
// instruction, into the fp32 dK rows. In deterministic mode (section "确定性计算": bitwise
// repeatable results) the records carry dI as 64-bit fixed point, a run that is the only
// contribution to its key rows is stored, and the pieces of a run cut by the CTA ranges go
// to a per-CTA scratch that km_det_combine sums in CTA order.
//
// A stage's data sit in three rings, each freed by its own consumer, so that the loads run
// ahead of the tensor cores by as many stages as their ring holds:
//   q ring      qw of the stage's rows (TMA), freed by the MMA (tcgen05.commit)
//   record ring the rows' records (bulk copy), freed by the dS builders once read
//   dS ring     the dS tile, written by the builders, freed by the MMA
//
// Warp roles (768 threads):
//   warp 0      q producer: for each row of a stage a TMA of qw_t (128-byte swizzle, zero
//               heads past N1), issued by lane 0
//   warp 1      MMA issuer and TMEM owner
//   warp 2      record producer: a bulk copy of each row's 256 records of the pair (lane 0)
//   warp 3      idle
//   warps 4-7   flush: finished dK^T buffers from TMEM to the fp32 key rows
//   warps 8-23  dS builders: two threads per key of the pair, each writing half of its
//               K-major row (contraction indices contiguous) with the 128-byte swizzle
//
// Every mbarrier wait is bounded; on expiry the CTA sets SLIKL_DEV_WAIT_TIMEOUT, the roles
// stop, in-flight copies and MMAs are waited for (again bounded), TMEM is freed.
#include <type_traits>

#include "slikl_sm100.cuh"

namespace slikl {
namespace {

using namespace sm100;

constexpr int kKmThreads = 768;
constexpr int kKmMaxQ = 4, kKmMaxR = 8, kKmDs = 2;   // ring slots (barrier arrays)
constexpr int kKmTmemCols = 512;         // two dK^T buffers of 256 columns

// Per instance: the query rows of a stage (G), its contraction width (G x N1P: 64, or 128
// with 128 heads), the largest record (mask words of the heads, dI; 8-byte records of
// N1 <= 32 grow to 16 in deterministic mode), the slots of the q and record rings, and the
// dS tile of a stage ([256 keys x contraction] as 64-wide column blocks of 256 x 128 B)
template <int N1P> __host__ __device__ constexpr int km_group() { return N1P < 64 ? 64 / N1P : 1; }
template <int N1P> __host__ __device__ constexpr int km_kdim() { return km_group<N1P>() * N1P; }
template <int N1P> __host__ __device__ constexpr int km_rec_bytes() { return N1P > 64 ? 32 : 16; }
template <int N1P> __host__ __device__ constexpr int km_q_slots() { return N1P > 64 ? 2 : 4; }
template <int N1P> __host__ __device__ constexpr int km_rec_slots() {
    return N1P > 64 ? 3 : (N1P < 32 ? 5 : 8);
}
template <int N1P> __host__ __device__ constexpr uint32_t km_ds_bytes() {
    return N1P > 64 ? 2u * 256u * 128u : 256u * 128u;
}

struct KmBarriers {
    uint64_t qfull[kKmMaxQ];             // q landed (TMA bytes)
    uint64_t qempty[kKmMaxQ];            // q read by the MMA (tcgen05.commit)
    uint64_t rfull[kKmMaxR];             // records landed (bulk-copy bytes)
    uint64_t rempty[kKmMaxR];            // records read (16 builder warps)
    uint64_t dsr[kKmDs];                 // dS tile written (16 builder warps)
    uint64_t dsempty[kKmDs];             // dS tile read by the MMA (tcgen05.commit)
    uint64_t accf[2];                    // dK^T buffer complete (tcgen05.commit)
    uint64_t acce[2];                    // dK^T buffer flushed (4 flush warps)
    uint64_t drain;
};

struct KmPlan {
    uint32_t q, ds, rec, rec_slot, bar, total;
};

__host__ __device__ constexpr uint32_t round_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <int N1P>
__host__ __device__ constexpr KmPlan km_plan() {
    // [q slot][2 column blocks][KD contraction rows][128 B] | [dS slot][dS tile] |
    // [record slot][G rows][256 records] | barriers
    constexpr uint32_t RB = km_rec_bytes<N1P>(), DS = km_ds_bytes<N1P>();
    constexpr uint32_t KD = km_kdim<N1P>(), G = km_group<N1P>();
    constexpr uint32_t kQ = km_q_slots<N1P>() * KD * 256u, kD = kKmDs * DS;
    constexpr uint32_t kSlot = G * 256u * RB;
    constexpr uint32_t kR = km_rec_slots<N1P>() * kSlot;
    return KmPlan{0u,
                  kQ,
                  kQ + kD,
                  kSlot,
                  round_up(kQ + kD + kR, 8),
                  round_up(kQ + kD + kR, 8) + (uint32_t)sizeof(KmBarriers) + 1024u};
}

struct KmItem {
    int t;           // query row
    int key0;        // first key row of the pair (identifies the run)
    int kloc;        // first key of the pair within the batch's key range
    int nkeys;       // keys of the pair inside the batch's key range
    bool first;      // first row of a run
    bool last;       // last row of a run
};

// The item sequence of a CTA: every set bit of every unit in [u0, u1), in order. Every role
// walks it on its own.
struct KmIter {
    const int4 *U;
    int u, u1;
    int4 cu, nu;
    uint32_t m;
    bool has_nu;
    int prev_key0;

    __device__ void find_next(int from) {
        has_nu = false;
        for (int k = from; k < u1; ++k) {
            const int4 x = U[k];
            if (x.w) { nu = x; u = k; has_nu = true; return; }
        }
        u = u1;
    }
    __device__ void init(const int4 *units, int a, int b) {
        U = units; u1 = b; prev_key0 = -1; m = 0;
        find_next(a);
        if (has_nu) {
            cu = nu;
            m = (uint32_t)cu.w;
            find_next(u + 1);
        }
    }
    __device__ bool next(KmItem &it) {
        if (!m) return false;
        const int bit = __ffs((int)m) - 1;
        m &= m - 1;
        it.t = cu.x + bit;
        it.key0 = cu.y;
        it.kloc = cu.z & 0xFFFF;
        it.nkeys = (int)((uint32_t)cu.z >> 16);
        it.first = cu.y != prev_key0;
        prev_key0 = cu.y;
        if (m == 0) {
            if (has_nu) {
                it.last = nu.y != cu.y;
                cu = nu;
                m = (uint32_t)cu.w;
                find_next(u + 1);
            } else {
                it.last = true;
            }
        } else {
            it.last = false;
        }
        return true;
    }
};

// The rows of one stage: up to G consecutive items of one run (a stage ends at its run's
// last item), taken in the order of KmIter by every role alike.
template <int G>
struct KmGroup {
    int t[G];        // query rows
    int n;           // rows present, 1..G
    int key0, kloc, nkeys;
    bool first;      // starts a run
    bool last;       // ends a run

    __device__ bool next(KmIter &iter) {
        n = 0;
        bool open = true;
#pragma unroll
        for (int j = 0; j < G; ++j) {
            KmItem it;
            if (open && iter.next(it)) {
                if (j == 0) {
                    key0 = it.key0; kloc = it.kloc; nkeys = it.nkeys; first = it.first;
                }
                t[j] = it.t;
                n = j + 1;
                last = it.last;
                open = !it.last;
            } else {
                open = false;
            }
        }
        return n > 0;
    }
    // query row of contraction row block r (r < G)
    __device__ int row(int r) const {
        int v = t[0];
#pragma unroll
        for (int j = 1; j < G; ++j)
            if (r == j) v = t[j];
        return v;
    }
};

template <int N1P, int D, typename T>
__global__ void __launch_bounds__(kKmThreads, 1)
    dk_keymajor(Params P, const __grid_constant__ CUtensorMap qmap) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int RB = km_rec_bytes<N1P>();
    constexpr int kG = km_group<N1P>();                          // query rows per stage
    constexpr int KD = km_kdim<N1P>();                           // contraction width of a stage
    constexpr int kSQ = km_q_slots<N1P>();                      // q ring slots
    constexpr int kSR = km_rec_slots<N1P>();                    // record ring slots
    constexpr uint32_t kDs = km_ds_bytes<N1P>();
    constexpr KmPlan SP = km_plan<N1P>();
    constexpr int kFmt = std::is_same<T, __nv_bfloat16>::value ? 1 : 0;
    constexpr uint32_t kIdesc = idesc_f16(kFmt, 128, 256, 1, 0);
    const int rb = P.rec_bytes;                                  // record bytes of this call
    constexpr uint32_t kQRow = (D / 64) * N1P * 128;            // q boxes of a row
    KmBarriers *bars = reinterpret_cast<KmBarriers *>(smem + SP.bar);
    __shared__ volatile int abort_flag;
    __shared__ uint32_t tmem_base;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u0 = P.km_range[blockIdx.x], u1 = P.km_range[blockIdx.x + 1];

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < kSQ; ++s) {
            mbar_init(&bars->qfull[s], 1);
            mbar_init(&bars->qempty[s], 1);
        }
        for (int s = 0; s < kSR; ++s) {
            mbar_init(&bars->rfull[s], 1);
            mbar_init(&bars->rempty[s], 16);
        }
        for (int s = 0; s < kKmDs; ++s) {
            mbar_init(&bars->dsr[s], 16);
            mbar_init(&bars->dsempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->accf[b], 1);
            mbar_init(&bars->acce[b], 4);
        }
        mbar_init(&bars->drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (D == 64) {
        // the upper column block of every q slot stays zero (rows d >= 64 of q^T)
        for (uint32_t i = threadIdx.x; i < kSQ * KD * 128 / 16; i += kKmThreads) {
            const uint32_t st = i / (KD * 8), r = i % (KD * 8);
            reinterpret_cast<uint4 *>(smem + SP.q + st * KD * 256 + KD * 128)[r] =
                make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&tmem_base)), "r"(kKmTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tacc = tmem_base;

    KmIter iter;
    iter.init(P.units_c, u0, u1);
    KmGroup<kG> grp;

    if (warp == 0) {
        // =============================== q producer ===============================
        uint32_t i = 0;
        bool ok = true;
        while (grp.next(iter)) {
            const int s = i % kSQ;
            if (!wait_bar(&bars->qempty[s], ((i / kSQ) & 1) ^ 1, &abort_flag, P.status)) { ok = false; break; }
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars->qfull[s], kQRow * (uint32_t)grp.n);
                const uint32_t qd = smem_u32(smem + SP.q + s * KD * 256);
#pragma unroll
                for (int r = 0; r < kG; ++r) {
                    if (r < grp.n) {
                        tma_load_3d(qd + r * N1P * 128, &qmap, 0, 0, grp.t[r], &bars->qfull[s]);
                        if (D == 128)
                            tma_load_3d(qd + KD * 128 + r * N1P * 128, &qmap, 64, 0, grp.t[r],
                                        &bars->qfull[s]);
                    }
                }
            }
            __syncwarp();
            ++i;
        }
        if (!ok && lane == 0) {
            // wait (bounded) for the copies already issued before the CTA leaves
            for (uint32_t j = i > kSQ ? i - kSQ : 0; j < i; ++j) {
                const long long st = clock64();
                while (!mbar_try_wait(&bars->qfull[j % kSQ], (j / kSQ) & 1) &&
                       clock64() - st < kWaitCycles) {}
            }
        }
    } else if (warp == 2) {
        // ============================= record producer =============================
        // the rows' records by bulk copy, issued by lane 0
        uint32_t i = 0;
        bool ok = true;
        while (grp.next(iter)) {
            const int s = i % kSR;
            if (!wait_bar(&bars->rempty[s], ((i / kSR) & 1) ^ 1, &abort_flag, P.status)) { ok = false; break; }
            if (lane == 0) {
                uint8_t *slot = smem + SP.rec + s * SP.rec_slot;
                mbar_arrive_expect_tx(&bars->rfull[s], 256u * (uint32_t)rb * (uint32_t)grp.n);
#pragma unroll
                for (int r = 0; r < kG; ++r) {
                    if (r < grp.n)
                        bulk_g2s(smem_u32(slot + r * 256 * RB),
                                 static_cast<const char *>(P.rec) +
                                     ((int64_t)grp.t[r] * P.S2m + grp.kloc) * rb,
                                 256 * rb, &bars->rfull[s]);
                }
            }
            __syncwarp();
            ++i;
        }
        if (!ok && lane == 0) {
            for (uint32_t j = i > kSR ? i - kSR : 0; j < i; ++j) {
                const long long st = clock64();
                while (!mbar_try_wait(&bars->rfull[j % kSR], (j / kSR) & 1) &&
                       clock64() - st < kWaitCycles) {}
            }
        }
    } else if (warp == 1) {
        // =============================== MMA issuer ===============================
        uint32_t i = 0, nrun = 0;
        while (grp.next(iter)) {
            const int sq = i % kSQ, sd = i % kKmDs;
            const int ab = nrun & 1;
            if (!wait_bar(&bars->qfull[sq], (i / kSQ) & 1, &abort_flag, P.status)) break;
            if (!wait_bar(&bars->dsr[sd], (i / kKmDs) & 1, &abort_flag, P.status)) break;
            if (grp.first && !wait_bar(&bars->acce[ab], ((nrun >> 1) & 1) ^ 1, &abort_flag, P.status)) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t qa = smem_u32(smem + SP.q + sq * KD * 256);
                const uint32_t da = smem_u32(smem + SP.ds + sd * kDs);
                const int nks = grp.n * (N1P / 16);   // 16-wide contraction steps of the rows present
#pragma unroll
                for (int ks = 0; ks < KD / 16; ++ks) {
                    if (ks < nks) {
                        const uint64_t a = sdesc(qa + ks * 2048, KD * 128, 1024);   // q^T, MN-major
                        // dS, K-major: 16 contraction indices per step, 64-wide column blocks
                        // of 256 rows
                        const uint64_t b = sdesc(da + (ks >> 2) * (256 * 128) + (ks & 3) * 32, 16, 1024);
                        umma_f16(tacc + ab * 256, a, b, kIdesc, (grp.first && ks == 0) ? 0u : 1u);
                    }
                }
                umma_commit(&bars->qempty[sq]);
                umma_commit(&bars->dsempty[sd]);
                if (grp.last) umma_commit(&bars->accf[ab]);
            }
            __syncwarp();
            if (grp.last) ++nrun;
            ++i;
        }
        if (lane == 0) umma_commit(&bars->drain);
        __syncwarp();
        const long long st = clock64();
        while (!mbar_try_wait(&bars->drain, 0) && clock64() - st < kWaitCycles) {}
    } else if (warp >= 4 && warp < 8) {
        // =============================== flush ===============================
        const int quad = warp & 3;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        // deterministic mode: a run is the only contribution to its key rows, stored as it is,
        // unless this CTA's unit range cuts it (the first run, continued from the previous
        // range: scratch slot 0; the last, continued by the next range: slot 1); the pieces of
        // a cut run are summed in CTA order by km_det_combine
        const bool det = P.deterministic != 0;
        const int n_units = P.km_range[gridDim.x];
        const bool cut_head = det && u0 < u1 && u0 > 0 && P.units_c[u0].y == P.units_c[u0 - 1].y;
        const bool cut_tail = det && u0 < u1 && u1 < n_units && P.units_c[u1].y == P.units_c[u1 - 1].y;
        const int head_key = u0 < u1 ? P.units_c[u0].y : -1;
        const int tail_key = u0 < u1 ? P.units_c[u1 - 1].y : -1;
        uint32_t nrun = 0;
        while (grp.next(iter)) {
            if (!grp.last) continue;
            const int ab = nrun & 1;
            if (!wait_bar(&bars->accf[ab], (nrun >> 1) & 1, &abort_flag, P.status)) break;
            tc_fence_after();
            if (quad * 32 < D) {
                float *dst = P.dk_acc + (int64_t)grp.key0 * D;
                if (cut_head && grp.key0 == head_key)
                    dst = P.km_scratch + (int64_t)(2 * blockIdx.x) * 256 * D;
                else if (cut_tail && grp.key0 == tail_key)
                    dst = P.km_scratch + (int64_t)(2 * blockIdx.x + 1) * 256 * D;
                dst += quad * 32 + lane;
#pragma unroll 1
                for (int c = 0; c < 256; c += 32) {
                    if (c >= grp.nkeys) break;
                    float v[32];
                    tmem_ld32(tacc + ab * 256 + lane_addr + c, v);
                    tmem_wait_ld();
                    if (det) {
#pragma unroll
                        for (int k = 0; k < 32; ++k)
                            if (c + k < grp.nkeys) dst[(int64_t)(c + k) * D] = v[k];
                    } else {
#pragma unroll
                        for (int k = 0; k < 32; ++k)
                            if (c + k < grp.nkeys) red_add_f32(dst + (int64_t)(c + k) * D, v[k]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acce[ab]);
            ++nrun;
        }
    } else if (warp >= 8) {
        // =============================== dS builders ===============================
        // two threads per key of the pair, each writing half of its K-major row: 32
        // contraction indices (64 with 128 heads), i.e. two rows of 16 heads, one row of 32, or
        // half the heads of one row of 64 or 128
        const int e = (threadIdx.x - 256) >> 1;   // key of the pair, 0..255
        const int half = threadIdx.x & 1;
        constexpr int kPer = KD / 16;             // 16-byte chunks (8 contraction indices) per thread
        constexpr int kSpan = 8 * kPer;           // contraction indices per thread
        constexpr int kRowsPer = kSpan >= N1P ? kSpan / N1P : 1;   // query rows per thread
        constexpr int kChRow = kPer / kRowsPer;   // chunks per query row (at most 8: two mask words)
        const int c0 = half * kPer;               // first chunk of this thread
        const int g0 = (8 * c0) / N1P;            // its first query row of the stage
        const int hb = (8 * c0) % N1P;            // and the first head within that row
        // chunks held in registers until the dS slot is free, so that the record slot is
        // released early; with 128 heads (8 chunks a thread) the dS slot is awaited first and
        // the chunks are stored as they are formed
        constexpr bool kHold = kPer <= 4;
        uint32_t i = 0;
        while (grp.next(iter)) {
            const int sr = i % kSR, sd = i % kKmDs;
            if (!wait_bar(&bars->rfull[sr], (i / kSR) & 1, &abort_flag, P.status)) break;
            if (!kHold && !wait_bar(&bars->dsempty[sd], ((i / kKmDs) & 1) ^ 1, &abort_flag, P.status)) break;
            const uint8_t *slot = smem + SP.rec + sr * SP.rec_slot;
            uint8_t *row = smem + SP.ds + sd * kDs + e * 128;
            uint4 o[kRowsPer][kChRow];            // this thread's chunks, packed
#pragma unroll
            for (int rr = 0; rr < kRowsPer; ++rr) {
                const int g = g0 + rr;
                if (g < grp.n) {                  // the MMA reads the chunks of present rows only
                    const uint8_t *rp = slot + g * 256 * RB + e * rb;
                    const uint32_t *mw = reinterpret_cast<const uint32_t *>(rp) + hb / 32;
                    const uint32_t m0 = mw[0];    // mask bits of this thread's heads
                    const uint32_t m1 = kChRow > 4 ? mw[1] : 0u;
                    const uint8_t *dp = rp + rec_di_offset(rb);
                    const float dI = P.deterministic
                                         ? di_from_fixed(*reinterpret_cast<const long long *>(dp))
                                         : *reinterpret_cast<const float *>(dp);
                    const uint32_t hh = pack2<T>(dI, dI);   // dI rounded to T, in both halves
#pragma unroll
                    for (int j = 0; j < kChRow; ++j) {   // 8 heads = one 16-byte chunk
                        const int c = c0 + rr * kChRow + j;
                        const uint32_t mb = ((j < 4 ? m0 : m1) >> ((j & 3) * 8)) & 0xFFu;
                        uint32_t wd[4];                  // heads 2k, 2k + 1: dI where S > 0, else +0
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t lo = 0u - ((mb >> (2 * k)) & 1u);
                            const uint32_t hi = 0u - ((mb >> (2 * k + 1)) & 1u);
                            wd[k] = hh & ((lo & 0xFFFFu) | (hi & 0xFFFF0000u));
                        }
                        const uint4 v = make_uint4(wd[0], wd[1], wd[2], wd[3]);
                        if (kHold)
                            o[rr][j] = v;
                        else   // chunk of the K-major row; column block c / 8
                            *reinterpret_cast<uint4 *>(row + (c >> 3) * (256 * 128) + ((((c & 7) ^ e) & 7) << 4)) = v;
                    }
                }
            }
            // the records of this slot are read (their values are in registers)
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->rempty[sr]);
            if (kHold && !wait_bar(&bars->dsempty[sd], ((i / kKmDs) & 1) ^ 1, &abort_flag, P.status)) break;
#pragma unroll
            for (int rr = 0; rr < kRowsPer; ++rr) {
                if (kHold && g0 + rr < grp.n) {
#pragma unroll
                    for (int j = 0; j < kChRow; ++j) {
                        const int c = c0 + rr * kChRow + j;   // chunk of the K-major row; column block c / 8
                        *reinterpret_cast<uint4 *>(row + (c >> 3) * (256 * 128) + ((((c & 7) ^ e) & 7) << 4)) = o[rr][j];
                    }
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->dsr[sd]);
            ++i;
        }
    }

    // ---------------- teardown ----------------
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tacc),
                     "r"(kKmTmemCols));
    }
}

// Deterministic mode: the 256-key block pairs whose run of units the CTA ranges cut. Block c
// starts a chain when its last run goes on into the next range and began inside its own; the
// pieces (c's last run, then the first run of each following non-empty range while the run
// goes on) are summed in that order into the fp32 key rows, which no other piece touches.
// Grid: (workers, 16); blockIdx.y takes 16 of the pair's 256 keys.
__global__ void km_det_combine(Params P, int workers) {
    __shared__ int chain[kKmDetWorkers];
    __shared__ int nchain;
    const int c = blockIdx.x;
    const int u0 = P.km_range[c], u1 = P.km_range[c + 1], n = P.km_range[workers];
    if (u0 >= u1 || u1 >= n) return;
    const int key0 = P.units_c[u1 - 1].y;
    if (P.units_c[u1].y != key0) return;                       // the last run ends here
    if (u0 > 0 && P.units_c[u0].y == key0 && P.units_c[u0 - 1].y == key0) return;  // began before
    if (threadIdx.x == 0) {
        int m = 0;
        for (int c2 = c + 1; c2 < workers; ++c2) {
            const int a = P.km_range[c2], b = P.km_range[c2 + 1];
            if (a >= b) continue;                               // empty range
            chain[m++] = c2;                                    // its first run goes on with ours
            if (!(P.units_c[b - 1].y == key0 && b < n && P.units_c[b].y == key0)) break;
        }
        nchain = m;
    }
    __syncthreads();
    const int nkeys = (int)((uint32_t)P.units_c[u1 - 1].z >> 16);
    const int kend = 16 * ((int)blockIdx.y + 1) < nkeys ? 16 * ((int)blockIdx.y + 1) : nkeys;
    const int64_t piece = (int64_t)256 * P.D;
    const float *first = P.km_scratch + (2 * (int64_t)c + 1) * piece;
    for (int e = 16 * (int)blockIdx.y * P.D + threadIdx.x; e < kend * P.D; e += blockDim.x) {
        float acc = first[e];
        for (int m = 0; m < nchain; ++m) acc += P.km_scratch[2 * (int64_t)chain[m] * piece + e];
        P.dk_acc[(int64_t)key0 * P.D + e] = acc;
    }
}

// qw = w . q per (row, head), the fp32 product rounded to T (round to nearest even); 8
// elements per thread (q rows are 16-byte aligned, D a multiple of 8).
template <typename T>
__global__ void km_scale_q(Params P) {
    const int64_t per_row = P.D / 8;
    const int64_t n = (int64_t)P.T1 * P.N1 * per_row;
    const uint4 *src = static_cast<const uint4 *>(P.q);
    uint4 *dst = static_cast<uint4 *>(P.km_qw);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float wv = P.w[i / per_row];               // row index t * N1 + h
        const uint4 v = src[i];
        const uint32_t in[4] = {v.x, v.y, v.z, v.w};
        uint32_t out[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = unpack2<T>(in[k]);
            out[k] = pack2<T>(wv * f.x, wv * f.y);
        }
        dst[i] = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

template <int N1P, int D, typename T>
cudaError_t launch_km_t(const Params &P, int workers, cudaStream_t s) {
    constexpr KmPlan sp = km_plan<N1P>();
    static_assert(sp.total <= 227 * 1024, "key-major kernel shared memory");
    static_assert(km_q_slots<N1P>() <= kKmMaxQ && km_rec_slots<N1P>() <= kKmMaxR, "ring slots");
    km_scale_q<T><<<8 * 148, 256, 0, s>>>(P);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // the MMA's A operand is qw, laid out as q
    Params Pw = P;
    Pw.q = P.km_qw;
    CUtensorMap qmap;
    e = encode_q_map<N1P, T>(Pw, &qmap);
    if (e != cudaSuccess) return e;
    auto k = dk_keymajor<N1P, D, T>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total);
    if (e != cudaSuccess) return e;
    k<<<workers, kKmThreads, sp.total, s>>>(P, qmap);
    return cudaGetLastError();
}

template <int N1P, int D>
cudaError_t launch_km_d(const Params &P, int workers, cudaStream_t s) {
    return P.dtype == SLIKL_BF16 ? launch_km_t<N1P, D, __nv_bfloat16>(P, workers, s)
                                 : launch_km_t<N1P, D, __half>(P, workers, s);
}

template <int N1P>
cudaError_t launch_km_n(const Params &P, int workers, cudaStream_t s) {
    return P.D == 128 ? launch_km_d<N1P, 128>(P, workers, s) : launch_km_d<N1P, 64>(P, workers, s);
}

}  // namespace

cudaError_t launch_km_det_combine(const Params &P, int workers, cudaStream_t s) {
    if (workers > kKmDetWorkers) return cudaErrorInvalidValue;
    km_det_combine<<<dim3(workers, 16), 256, 0, s>>>(P, workers);
    return cudaGetLastError();
}

// Shapes: N1 <= 128, D in {64, 128}.
cudaError_t launch_dk_keymajor(const Params &P, int workers, cudaStream_t s) {
    if (P.N1 > 128 || (P.D != 64 && P.D != 128)) return cudaErrorInvalidValue;
    if (P.N1 <= 16) return launch_km_n<16>(P, workers, s);
    if (P.N1 <= 32) return launch_km_n<32>(P, workers, s);
    if (P.N1 <= 64) return launch_km_n<64>(P, workers, s);
    return launch_km_n<128>(P, workers, s);
}

}  // namespace slikl
