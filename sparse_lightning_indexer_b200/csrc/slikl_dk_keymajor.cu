// Key-major dK on the sm_100a tensor cores (tcgen05 MMA, accumulators in TMEM).
//
// The operator adds dK_topk(t) = dS_t^T . q_t into the key rows named by each query row t
// (aclnnSparseLightningIndexerKLLossGrad, section "计算公式"). Grouped by key instead of by
// query row, the same sum reads
//
//   dK_j = sum over the rows t that name key j of  sum_h dS_t[h, j] q_t[h, :]
//
// The fused kernel leaves one record per named (t, j): dI_tj and the set of heads with
// S_tjh > 0. dS_tjh = dI_tj * w_th * [S_tjh > 0] is rebuilt from it here (the same fp32
// product and rounding as the fused kernel's dS), and for one 256-key block pair the
// products of all rows that name a key of the pair accumulate in TMEM:
//
//   dK^T [D x 256 keys] += q_t^T [D x heads] . dS_t [heads x 256 keys]   (M = 128, N = 256)
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
// Warp roles (768 threads):
//   warp 0      producer: per stage, for each of its query rows a TMA of q_t (128-byte
//               swizzle, zero heads past N1) and a bulk copy of the pair's 256 records
//               (lane 0); w_t through registers
//   warp 1      MMA issuer and TMEM owner
//   warps 2-3   idle
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
constexpr int kKmStages = 4;             // most stages of any instance (barrier arrays)
constexpr int kKmTmemCols = 512;         // two dK^T buffers of 256 columns

// Per instance: the query rows of a stage (G), its contraction width (G x N1P: 64, or 128
// with 128 heads), the largest record (mask words of the heads, dI; 8-byte records of
// N1 <= 32 grow to 16 in deterministic mode), stages, and the dS tile of a stage ([256 keys x
// contraction] as 64-wide column blocks of 256 x 128 B)
template <int N1P> __host__ __device__ constexpr int km_group() { return N1P < 64 ? 64 / N1P : 1; }
template <int N1P> __host__ __device__ constexpr int km_kdim() { return km_group<N1P>() * N1P; }
template <int N1P> __host__ __device__ constexpr int km_rec_bytes() { return N1P > 64 ? 32 : 16; }
template <int N1P> __host__ __device__ constexpr int km_stages() {
    return N1P > 64 ? 2 : (N1P < 64 ? 3 : kKmStages);
}
template <int N1P> __host__ __device__ constexpr uint32_t km_ds_bytes() {
    return N1P > 64 ? 2u * 256u * 128u : 256u * 128u;
}

struct KmBarriers {
    uint64_t full[kKmStages];            // q, w, records landed (producer, TMA bytes)
    uint64_t dsr[kKmStages];             // dS tile written (16 builder warps)
    uint64_t empty[kKmStages];           // stage consumed by the MMA (tcgen05.commit)
    uint64_t accf[2];                    // dK^T buffer complete (tcgen05.commit)
    uint64_t acce[2];                    // dK^T buffer flushed (4 flush warps)
    uint64_t drain;
};

struct KmPlan {
    uint32_t q, ds, rec, w, bar, total;
};

__host__ __device__ constexpr uint32_t round_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <int N1P>
__host__ __device__ constexpr KmPlan km_plan() {
    // [stage][2 column blocks][KD contraction rows][128 B] | [stage][dS tile] |
    // [stage][G rows][256 records] | [stage][KD] | barriers
    constexpr uint32_t S = km_stages<N1P>(), RB = km_rec_bytes<N1P>(), DS = km_ds_bytes<N1P>();
    constexpr uint32_t KD = km_kdim<N1P>(), G = km_group<N1P>();
    constexpr uint32_t kQ = S * KD * 256u, kR = S * G * 256u * RB;
    return KmPlan{0u,
                  kQ,
                  kQ + S * DS,
                  kQ + S * DS + kR,
                  round_up(kQ + S * DS + kR + S * KD * 4u, 8),
                  round_up(kQ + S * DS + kR + S * KD * 4u, 8) + (uint32_t)sizeof(KmBarriers) +
                      1024u};
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
    constexpr int kSt = km_stages<N1P>();
    constexpr uint32_t kDs = km_ds_bytes<N1P>();
    constexpr KmPlan SP = km_plan<N1P>();
    constexpr int kFmt = std::is_same<T, __nv_bfloat16>::value ? 1 : 0;
    constexpr uint32_t kIdesc = idesc_f16(kFmt, 128, 256, 1, 0);
    const int rb = P.rec_bytes;                                  // record bytes of this call
    const uint32_t kTxRow = (D / 64) * N1P * 128 + 256 * rb;    // q boxes + records of a row
    KmBarriers *bars = reinterpret_cast<KmBarriers *>(smem + SP.bar);
    __shared__ volatile int abort_flag;
    __shared__ uint32_t tmem_base;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u0 = P.km_range[blockIdx.x], u1 = P.km_range[blockIdx.x + 1];

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < kSt; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->dsr[s], 16);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->accf[b], 1);
            mbar_init(&bars->acce[b], 4);
        }
        mbar_init(&bars->drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (D == 64) {
        // the upper column block of every q stage stays zero (rows d >= 64 of q^T)
        for (uint32_t i = threadIdx.x; i < kSt * KD * 128 / 16; i += kKmThreads) {
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
        // =============================== producer ===============================
        // w of the stage's rows goes through registers (its rows need only 4-byte alignment),
        // loaded one stage ahead; q_t and the records by TMA / bulk copy, issued by lane 0
        auto load_w = [&](const KmGroup<kG> &g, float *wv) {
#pragma unroll
            for (int k = 0; k < KD / 32; ++k) {
                const int c = lane + 32 * k;          // contraction index: row c / N1P, head c % N1P
                const int r = c / N1P, h = c % N1P;
                wv[k] = (r < g.n && h < P.N1) ? P.w[(int64_t)g.row(r) * P.N1 + h] : 0.f;
            }
        };
        float wcur[KD / 32], wnxt[KD / 32];
        uint32_t i = 0;
        bool ok = true, have = grp.next(iter);
        if (have) load_w(grp, wcur);
        while (have) {
            KmGroup<kG> nx;
            const bool have_nx = nx.next(iter);
            if (have_nx) load_w(nx, wnxt);
            const int s = i % kSt;
            if (!wait_bar(&bars->empty[s], ((i / kSt) & 1) ^ 1, &abort_flag, P.status)) { ok = false; break; }
            float *wd = reinterpret_cast<float *>(smem + SP.w + s * KD * 4);
#pragma unroll
            for (int k = 0; k < KD / 32; ++k) wd[lane + 32 * k] = wcur[k];
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars->full[s], kTxRow * (uint32_t)grp.n);
                const uint32_t qd = smem_u32(smem + SP.q + s * KD * 256);
#pragma unroll
                for (int r = 0; r < kG; ++r) {
                    if (r < grp.n) {
                        const int t = grp.t[r];
                        tma_load_3d(qd + r * N1P * 128, &qmap, 0, 0, t, &bars->full[s]);
                        if (D == 128)
                            tma_load_3d(qd + KD * 128 + r * N1P * 128, &qmap, 64, 0, t, &bars->full[s]);
                        bulk_g2s(smem_u32(smem + SP.rec + (s * kG + r) * 256 * RB),
                                 static_cast<const char *>(P.rec) + ((int64_t)t * P.S2m + grp.kloc) * rb,
                                 256 * rb, &bars->full[s]);
                    }
                }
            }
            __syncwarp();
            ++i;
            grp = nx;
            have = have_nx;
#pragma unroll
            for (int k = 0; k < KD / 32; ++k) wcur[k] = wnxt[k];
        }
        if (!ok && lane == 0) {
            // wait (bounded) for the copies already issued before the CTA leaves
            for (uint32_t j = i > kSt ? i - kSt : 0; j < i; ++j) {
                const long long st = clock64();
                while (!mbar_try_wait(&bars->full[j % kSt], (j / kSt) & 1) &&
                       clock64() - st < kWaitCycles) {}
            }
        }
    } else if (warp == 1) {
        // =============================== MMA issuer ===============================
        uint32_t i = 0, nrun = 0;
        while (grp.next(iter)) {
            const int s = i % kSt;
            const int ab = nrun & 1;
            if (!wait_bar(&bars->dsr[s], (i / kSt) & 1, &abort_flag, P.status)) break;
            if (grp.first && !wait_bar(&bars->acce[ab], ((nrun >> 1) & 1) ^ 1, &abort_flag, P.status)) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t qa = smem_u32(smem + SP.q + s * KD * 256);
                const uint32_t da = smem_u32(smem + SP.ds + s * kDs);
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
                umma_commit(&bars->empty[s]);
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
        uint32_t i = 0;
        while (grp.next(iter)) {
            const int s = i % kSt;
            if (!wait_bar(&bars->full[s], (i / kSt) & 1, &abort_flag, P.status)) break;
            const float *ws = reinterpret_cast<const float *>(smem + SP.w + s * KD * 4);
            uint8_t *row = smem + SP.ds + s * kDs + e * 128;
#pragma unroll
            for (int rr = 0; rr < kRowsPer; ++rr) {
                const int g = g0 + rr;
                if (g < grp.n) {                  // the MMA reads the chunks of present rows only
                    const uint8_t *rp = smem + SP.rec + (s * kG + g) * 256 * RB + e * rb;
                    const uint32_t *mw = reinterpret_cast<const uint32_t *>(rp) + hb / 32;
                    const uint32_t m0 = mw[0];    // mask bits of this thread's heads
                    const uint32_t m1 = kChRow > 4 ? mw[1] : 0u;
                    const uint8_t *dp = rp + rec_di_offset(rb);
                    const float dI = P.deterministic
                                         ? di_from_fixed(*reinterpret_cast<const long long *>(dp))
                                         : *reinterpret_cast<const float *>(dp);
#pragma unroll
                    for (int j = 0; j < kChRow; ++j) {   // 8 heads = one 16-byte chunk
                        const int c = c0 + rr * kChRow + j;   // chunk of the K-major row; column block c / 8
                        const float4 wa = *reinterpret_cast<const float4 *>(ws + 8 * c);
                        const float4 wb = *reinterpret_cast<const float4 *>(ws + 8 * c + 4);
                        const uint32_t mb = ((j < 4 ? m0 : m1) >> ((j & 3) * 8)) & 0xFFu;
                        const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
                        float d[8];
#pragma unroll
                        for (int h = 0; h < 8; ++h) d[h] = ((mb >> h) & 1u) ? dI * wv[h] : 0.f;
                        const uint4 o = make_uint4(pack2<T>(d[0], d[1]), pack2<T>(d[2], d[3]),
                                                   pack2<T>(d[4], d[5]), pack2<T>(d[6], d[7]));
                        *reinterpret_cast<uint4 *>(row + (c >> 3) * (256 * 128) + ((((c & 7) ^ e) & 7) << 4)) = o;
                    }
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->dsr[s]);
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

template <int N1P, int D, typename T>
cudaError_t launch_km_t(const Params &P, int workers, cudaStream_t s) {
    constexpr KmPlan sp = km_plan<N1P>();
    static_assert(sp.total <= 227 * 1024, "key-major kernel shared memory");
    CUtensorMap qmap;
    cudaError_t e = encode_q_map<N1P, T>(P, &qmap);
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
