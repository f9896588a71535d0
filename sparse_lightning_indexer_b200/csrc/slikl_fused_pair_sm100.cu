// Fused per-token kernel, record mode, with items of two slot tiles (256 slots).
//
// The same computation as the record mode of slikl_fused_sm100.cu
// (aclnnSparseLightningIndexerKLLossGrad, section "计算公式": S = q K_topk^T, I = W ReLU(S),
// y = Softmax(I), dI = y - p, dW = dI ReLU(S)^T, dq = dS K_topk, and per named key a record
// of dI and the heads with S > 0 for the key-major dK kernel), for N1 <= 64. An item here
// covers the slot tiles 2i and 2i + 1 of a token: 256 key rows are gathered per K stage, two
// S products (M = 128 keys each) fill one S buffer, each softmax thread takes two slots, and
// the dq product runs over 256 keys. Every barrier hand-off, MMA issue and scheduler step is
// paid once per 256 slots instead of once per 128: on B200 the per-item cost of that skeleton
// (about 3,000 cycles) dominated the 128-slot kernel whatever the head count.
//
// Schedule: as the 128-slot kernel (pass A of the next token alternating with pass B of the
// current one), over the token's non-empty tile pairs.
//
// Warp roles (384 threads):
//   warps 0-2, 4-7  producers: cp.async gather of the 256 key rows (16-byte chunks, zero-fill
//                   for invalid slots); warp 0 also loads q by TMA
//   warp 3          MMA issuer (one thread) and TMEM owner
//   warps 8-11      softmax group: pass-A and pass-B epilogues for slots lrow and lrow + 128,
//                   records, dW, dq readback
//
// TMEM: S buffers [0, 4 N1P) (buffer b, half h at (2b + h) N1P), dq^T at 4 N1P, the per-slot
// dW partials at 5 N1P (both halves of a pair add into the same columns), and (rows of at
// most 4096 slots) the parked logits of two tokens at 6 N1P + 32 (ordinal % 2) + 2 pair + h,
// their slot indices 64 columns on. Shared memory: two K stages of 256 rows (two
// 128-row halves of two 64-column SW128 blocks), two q buffers, one dS tile [256 keys x 64
// heads] (two halves), the producers' index rings.
//
// Every wait on an mbarrier is bounded (about one second of SM clock); on expiry the CTA
// sets SLIKL_DEV_WAIT_TIMEOUT, every role stops, in-flight copies and MMAs are drained, TMEM
// is freed and the kernel returns.
#include <type_traits>

#include "slikl_sm100.cuh"

namespace slikl {
namespace {

using namespace sm100;

constexpr int kPThreads = 384;
constexpr int kPTmemCols = 512;
constexpr int kPStages = 2;
constexpr int kPHalfBytes = 128 * 256;           // 128 key rows x 128 d
constexpr int kPStageBytes = 2 * kPHalfBytes;    // 256 key rows
constexpr int kPDsBytes = 2 * 16384;             // dS tile [256 keys x 64 heads]
constexpr int kPRingSlot = 260;                  // 256 slot indices, key base, key count
constexpr int kPProd = 7;

struct PBarriers {
    uint64_t kv_full[kPStages], kv_empty[kPStages];
    uint64_t q_full[2], q_empty[2];
    uint64_t s_full[2], s_empty[2];
    uint64_t ds_full, ds_empty;           // the dS tile: softmax group -> MMA -> softmax group
    uint64_t dq_full, dq_empty;
    uint64_t drain;
    uint64_t sm_sync;
};

struct PPlan {
    uint32_t kv, q, ds, w, red, ring, bar, total;
};

template <int N1P>
__host__ __device__ inline PPlan pair_plan() {
    PPlan s{};
    uint32_t off = 0;
    auto take = [&](uint32_t bytes, uint32_t align) {
        off = (off + align - 1) / align * align;
        const uint32_t o = off;
        off += bytes;
        return o;
    };
    s.kv = take(kPStages * kPStageBytes, 1024);
    s.q = take(2 * N1P * 256, 1024);
    s.ds = take(kPDsBytes, 1024);
    s.w = take(2 * N1P * 4, 16);
    s.red = take(2 * 4 * 64 * 4, 16);
    s.ring = take(kPProd * 4 * kPRingSlot * 4, 16);
    s.bar = take(sizeof(PBarriers) + 16, 8);
    s.total = off + 1024;
    return s;
}

struct PCtl {
    volatile int abort;
    uint32_t tmem_base;
    float stat_m[4], stat_z[4];
};

// bit i of the result: slot tile 2i or 2i + 1 of the 64-bit tile mask is non-empty
__device__ __forceinline__ uint64_t pair_mask(uint64_t m) {
    uint64_t x = (m | (m >> 1)) & 0x5555555555555555ull;
    x = (x | (x >> 1)) & 0x3333333333333333ull;
    x = (x | (x >> 2)) & 0x0f0f0f0f0f0f0f0full;
    x = (x | (x >> 4)) & 0x00ff00ff00ff00ffull;
    x = (x | (x >> 8)) & 0x0000ffff0000ffffull;
    x = (x | (x >> 16)) & 0x00000000ffffffffull;
    return x;
}

struct PItem {
    int kind;        // 0 = pass A, 1 = pass B, -1 = none
    int t;
    int pair;        // slots [256 pair, 256 pair + 256)
    int ord;
    bool first, last;
};

// The 128-slot kernel's schedule over tile pairs.
struct PSched {
    const uint64_t *tiles;
    int t_next, t_end;
    int ta, oa; uint64_t ma, ma_all; bool a_on, a_first, a_exists;
    int tb, ob; uint64_t mb; bool b_on, b_first;
    int next_ord;
    bool turn_b;

    __device__ bool find_a() {
        for (; t_next < t_end; ++t_next) {
            const uint64_t m = tiles[t_next];
            if (m) {
                ta = t_next++;
                oa = next_ord++;
                ma = ma_all = pair_mask(m);
                a_on = true;
                a_first = true;
                return true;
            }
        }
        a_on = false;
        return false;
    }
    __device__ void init(const uint64_t *tl, int t0, int t1) {
        tiles = tl; t_next = t0; t_end = t1; next_ord = 0;
        b_on = false; turn_b = true;
        a_exists = find_a();
    }
    __device__ PItem next() {
        PItem it;
        it.kind = -1;
        if (!a_on && !b_on) return it;
        const bool take_b = b_on && (!a_on || turn_b);
        turn_b = !turn_b;
        if (take_b) {
            it.kind = 1; it.t = tb; it.ord = ob; it.first = b_first;
            it.pair = __ffsll((long long)mb) - 1;
            mb &= mb - 1;
            it.last = mb == 0;
            b_first = false;
            if (it.last) b_on = false;
        } else {
            it.kind = 0; it.t = ta; it.ord = oa; it.first = a_first;
            it.pair = __ffsll((long long)ma) - 1;
            ma &= ma - 1;
            it.last = ma == 0;
            a_first = false;
            if (it.last) a_on = false;
        }
        if (!a_on && !b_on) {
            if (a_exists) { tb = ta; ob = oa; mb = ma_all; b_on = true; b_first = true; }
            a_exists = find_a();
            turn_b = true;
        }
        return it;
    }
};

// kMode: 1 = records with fp32 dI; 2 = deterministic (64-bit fixed-point dI, 16-byte records
// at least). kTP: the logits I of pass A are parked in TMEM (rows of at most 16 tile pairs,
// two tokens in flight: 64 columns) instead of in softmax_out, saving a global store and load
// per slot
template <int N1P, int D, typename T, int kMode, bool kTP>
__global__ void __launch_bounds__(kPThreads, 1)
    fused_pair_sm100(Params P, const __grid_constant__ CUtensorMap qmap) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int K = P.K;
    const PPlan SP = pair_plan<N1P>();
    PBarriers *bars = reinterpret_cast<PBarriers *>(smem + SP.bar);
    __shared__ PCtl ctl;
    constexpr int kFmt = std::is_same<T, __nv_bfloat16>::value ? 1 : 0;
    constexpr uint32_t kIdescS = idesc_f16(kFmt, 128, N1P, 0, 0);
    constexpr uint32_t kIdescDq = idesc_f16(kFmt, 128, N1P, 1, 1);
    constexpr int kDChunks = D / 8;
    constexpr int kC = N1P < 32 ? N1P : 32;
    constexpr int kRecBytes = N1P > 32 || kMode == 2 ? 16 : 8;
    constexpr uint32_t kColDq = 4 * N1P;
    constexpr uint32_t kColDw = 5 * N1P;
    static_assert(N1P <= 64, "paired items take at most 64 heads");
    static_assert(kColDw + N1P <= kPTmemCols, "TMEM columns");
    // the dW partials of both halves of a pair share columns (one thread holds both slots);
    // then the parked I [token ordinal % 2][32] and the parked slot indices, likewise
    constexpr uint32_t kColPark = kColDw + N1P;
    static_assert(!kTP || kColPark + 128 <= kPTmemCols, "TMEM columns (parked logits)");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = P.meta[kMetaHeader + 2 * blockIdx.x];
    const int t1 = P.meta[kMetaHeader + 2 * blockIdx.x + 1];

    // ---------------- setup ----------------
    if (threadIdx.x == 0) {
        ctl.abort = 0;
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&bars->kv_full[s], 32 * kPProd);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->q_full[b], 1);
            mbar_init(&bars->q_empty[b], 1);
            mbar_init(&bars->s_full[b], 1);
            mbar_init(&bars->s_empty[b], 4);
        }
        mbar_init(&bars->ds_full, 4);
        mbar_init(&bars->ds_empty, 1);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_empty, 4);
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->sm_sync, 4);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // heads past N1P of the dS tile, padded heads of q and (D = 64) the upper column block of
    // q and of every K stage half stay zero
    for (uint32_t i = threadIdx.x; i < kPDsBytes / 16; i += kPThreads)
        reinterpret_cast<uint4 *>(smem + SP.ds)[i] = make_uint4(0, 0, 0, 0);
    for (uint32_t i = threadIdx.x; i < (uint32_t)(2 * N1P * 256 / 16); i += kPThreads)
        reinterpret_cast<uint4 *>(smem + SP.q)[i] = make_uint4(0, 0, 0, 0);
    if (D == 64) {
        for (int s = 0; s < 2 * kPStages; ++s)
            for (uint32_t i = threadIdx.x; i < 16384 / 16; i += kPThreads)
                reinterpret_cast<uint4 *>(smem + SP.kv + s * kPHalfBytes + 16384)[i] =
                    make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async();
    if (warp == 3) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&ctl.tmem_base)), "r"(kPTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    const uint32_t tm_s = tmem;
    const uint32_t tm_dq = tmem + kColDq;
    const uint32_t tm_dw = tmem + kColDw;

    PSched sc;
    sc.init(P.tok_tiles, t0, t1);

    if (warp < 3 || (warp >= 4 && warp < 8)) {
        // =============================== producers ===============================
        // As the 128-slot kernel: every producer warp walks every item and waits on every
        // stage phase; each copies its share of the 256 rows; the slot indices, key base and
        // key count of an item are loaded four items ahead and kept in a 4-slot ring two
        // items ahead.
        const int rsub = lane / kDChunks;
        const int chunk = lane % kDChunks;
        constexpr int kRowsPerPass = 32 / kDChunks;
        const char *kbase_ptr = static_cast<const char *>(P.k);
        const int pw = warp < 3 ? warp : warp - 1;
        int32_t *ring = reinterpret_cast<int32_t *>(smem + SP.ring) + pw * 4 * kPRingSlot;
        bool ok = true;
        struct IdxRegs { int32_t v[8]; int32_t kb, kl; };
        auto ldg_idx = [&](const PItem &it, IdxRegs &r) {
            const int32_t *irow = P.idx + (int64_t)it.t * K;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = it.pair * 256 + lane + 32 * u;
                r.v[u] = j < K ? irow[j] : -1;
            }
            r.kb = P.tok_kbase[it.t];
            r.kl = P.tok_klen[it.t];
        };
        auto sts_idx = [&](const IdxRegs &r, int slot) {
            int32_t *d = ring + slot * kPRingSlot;
#pragma unroll
            for (int u = 0; u < 8; ++u) d[lane + 32 * u] = r.v[u];
            if (lane == 0) { d[256] = r.kb; d[257] = r.kl; }
        };
        PItem it0 = sc.next();
        PItem it1 = it0.kind >= 0 ? sc.next() : it0;
        PItem it2 = it1.kind >= 0 ? sc.next() : it1;
        PItem it3 = it2.kind >= 0 ? sc.next() : it2;
        IdxRegs r2{}, r3{};
        if (it0.kind >= 0) { IdxRegs r; ldg_idx(it0, r); sts_idx(r, 0); }
        if (it1.kind >= 0) { IdxRegs r; ldg_idx(it1, r); sts_idx(r, 1); }
        if (it2.kind >= 0) ldg_idx(it2, r2);
        if (it3.kind >= 0) ldg_idx(it3, r3);
        int q_last = -1;
        uint32_t g = 0;
        while (ok && it0.kind >= 0) {
            __syncwarp();
            if (warp == 0 && it0.kind == 0 && it0.first) {
                const int qb = it0.ord & 1;
                if (!wait_bar(&bars->q_empty[qb], ((it0.ord >> 1) & 1) ^ 1, &ctl.abort, P.status)) { ok = false; break; }
                if (lane == 0) {
                    const uint32_t qdst = smem_u32(smem + SP.q + qb * N1P * 256);
                    mbar_arrive_expect_tx(&bars->q_full[qb], (D / 64) * N1P * 128);
                    tma_load_3d(qdst, &qmap, 0, 0, it0.t, &bars->q_full[qb]);
                    if (D == 128) tma_load_3d(qdst + N1P * 128, &qmap, 64, 0, it0.t, &bars->q_full[qb]);
                }
                q_last = it0.ord;
            }
            const int s = g % kPStages;
            if (!wait_bar(&bars->kv_empty[s], ((g / kPStages) & 1) ^ 1, &ctl.abort, P.status)) { ok = false; break; }
            const int32_t *slot = ring + (g & 3) * kPRingSlot;
            const int32_t kb = slot[256], kl = slot[257];
            const int jbase = it0.pair * 256;
            const uint32_t dst0 = smem_u32(smem + SP.kv + s * kPStageBytes) + (chunk >> 3) * 16384;
            constexpr int kGroups = 256 / kRowsPerPass;
            constexpr int kPer = (kGroups + kPProd - 1) / kPProd;
            int32_t vv[kPer];
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int i = pw + kPProd * j;
                vv[j] = i < kGroups ? slot[rsub + kRowsPerPass * i] : -1;
            }
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int i = pw + kPProd * j;
                if (i < kGroups) {
                    const int r = rsub + kRowsPerPass * i;        // row of the pair, 0..255
                    const int32_t v = vv[j];
                    const bool valid = jbase + r < K && v >= 0 && v < kl;
                    const char *src = kbase_ptr + (valid ? ((int64_t)(kb + v) * (D * 2) + chunk * 16) : 0);
                    cp_async16(dst0 + (r >> 7) * kPHalfBytes + sw128(r & 127, (chunk & 7) * 8), src,
                               valid ? 16 : 0);
                }
            }
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&bars->kv_full[s]))
                         : "memory");
            if (it2.kind >= 0) sts_idx(r2, (g + 2) & 3);
            it0 = it1;
            it1 = it2;
            it2 = it3;
            r2 = r3;
            if (it3.kind >= 0) {
                it3 = sc.next();
                if (it3.kind >= 0) ldg_idx(it3, r3);
            }
            ++g;
        }
        cp_async_wait<0>();
        if (!ok && q_last >= 0 && lane == 0) {
            const long long st = clock64();
            while (!mbar_try_wait(&bars->q_full[q_last & 1], (q_last >> 1) & 1) &&
                   clock64() - st < kWaitCycles) {}
        }
    } else if (warp == 3) {
        // =============================== MMA issuer ===============================
        uint32_t gk = 0, gd = 0, nb = 0;
        bool ok = true;
        const uint32_t kv0 = smem_u32(smem + SP.kv);
        const uint32_t q0 = smem_u32(smem + SP.q);
        const uint32_t ds0 = smem_u32(smem + SP.ds);
        // S^T of both halves of item gk into S buffer gk % 2 (pass-A stages released right away)
        auto issue_s = [&](const PItem &it, int &stage) -> bool {
            const int s = gk % kPStages, b = gk & 1;
            const int qb = it.ord & 1;
            if (it.kind == 0 && it.first &&
                !wait_bar(&bars->q_full[qb], (it.ord >> 1) & 1, &ctl.abort, P.status)) return false;
            if (!wait_bar(&bars->kv_full[s], (gk / kPStages) & 1, &ctl.abort, P.status)) return false;
            if (!wait_bar(&bars->s_empty[b], ((gk >> 1) & 1) ^ 1, &ctl.abort, P.status)) return false;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t qaddr = q0 + qb * N1P * 256;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t kaddr = kv0 + s * kPStageBytes + h * kPHalfBytes;
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                        const uint32_t qoff = (ks >> 2) * (N1P * 128) + (ks & 3) * 32;
                        umma_f16(tm_s + (2 * b + h) * N1P, sdesc(kaddr + off, 16, 1024),
                                 sdesc(qaddr + qoff, 16, 1024), kIdescS, ks > 0);
                    }
                }
                umma_commit(&bars->s_full[b]);
                if (it.kind == 0) umma_commit(&bars->kv_empty[s]);
            }
            __syncwarp();
            stage = s;
            ++gk;
            return true;
        };
        PItem cur = sc.next();
        int st_cur = 0, st_nxt = 0;
        if (cur.kind >= 0 && !issue_s(cur, st_cur)) ok = false;
        while (ok && cur.kind >= 0) {
            const PItem nxt = sc.next();
            if (nxt.kind >= 0 && !issue_s(nxt, st_nxt)) { ok = false; break; }
            if (cur.kind == 1) {
                if (cur.first && !wait_bar(&bars->dq_empty, (nb & 1) ^ 1, &ctl.abort, P.status)) { ok = false; break; }
                if (!wait_bar(&bars->ds_full, gd & 1, &ctl.abort, P.status)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t kaddr = kv0 + st_cur * kPStageBytes;
#pragma unroll
                    for (int ks = 0; ks < 16; ++ks) {      // 256 keys, 16 per step
                        const uint64_t a = sdesc(kaddr + (ks >> 3) * kPHalfBytes + (ks & 7) * 2048, 16384, 1024);
                        const uint64_t bd = sdesc(ds0 + (ks >> 3) * 16384 + (ks & 7) * 2048, 16384, 1024);
                        umma_f16(tm_dq, a, bd, kIdescDq, (!cur.first || ks > 0) ? 1u : 0u);
                    }
                    umma_commit(&bars->kv_empty[st_cur]);
                    umma_commit(&bars->ds_empty);            // dS tile read by the dq product
                    if (cur.last) {
                        umma_commit(&bars->dq_full);
                        umma_commit(&bars->q_empty[cur.ord & 1]);
                    }
                }
                __syncwarp();
                if (cur.last) ++nb;
                ++gd;
            }
            cur = nxt;
            st_cur = st_nxt;
        }
        if (lane == 0) umma_commit(&bars->drain);
        __syncwarp();
        {
            const long long start = clock64();
            while (!mbar_try_wait(&bars->drain, 0) && clock64() - start < kWaitCycles) {}
        }
    } else if (warp >= 8) {
        // =============================== softmax group ===============================
        const int ew = warp - 8;
        const int quad = warp & 3;
        const int lrow = quad * 32 + lane;       // slot lrow of each half; d for dq
        const int et = threadIdx.x - 256;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        float *wsm = reinterpret_cast<float *>(smem + SP.w);
        float *red = reinterpret_cast<float *>(smem + SP.red);
        uint8_t *ds_tile = smem + SP.ds;
        uint32_t gk = 0, gd = 0, nb = 0, ph = 0;
        bool ok = true;
        for (int t = t0; t < t1; ++t) {
            if (P.tok_tiles[t]) continue;
            for (int j = et; j < K; j += 128) P.y[(int64_t)t * K + j] = 0.f;
            for (int e = et; e < P.N1 * D; e += 128)
                reinterpret_cast<T *>(P.dq)[(int64_t)t * P.N1 * D + e] = T(0.f);
            for (int h = et; h < P.N1; h += 128) P.dw[(int64_t)t * P.N1 + h] = 0.f;
        }
        float m_a = -INFINITY, z_a = 0.f;
        float M_n = -INFINITY, iZ_n = 0.f;
        float M_b = -INFINITY, iZ_b = 0.f;
        struct Pre { int32_t v[2], kl, kb; float p[2], I[2]; bool haveI; };
        auto prefetch = [&](const PItem &nx, const PItem &cu, Pre &o) {
            const int64_t ro = (int64_t)nx.t * K;
            o.kl = P.tok_klen[nx.t];
            o.kb = P.tok_kbase[nx.t];
            o.haveI = nx.kind == 1 && !(cu.kind == 0 && cu.t == nx.t && cu.pair == nx.pair);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int jn = nx.pair * 256 + h * 128 + lrow;
                // (pass-B slot indices come from the parked copy when parking)
                o.v[h] = (!(kTP && nx.kind == 1) && jn < K) ? P.idx[ro + jn] : -1;
                o.p[h] = (nx.kind == 1 && jn < K) ? P.p[ro + jn] : 0.f;
                o.I[h] = (!kTP && o.haveI && jn < K) ? P.y[ro + jn] : 0.f;
            }
        };
        PItem it = sc.next();
        Pre cur{};
        if (it.kind >= 0) {
            PItem none;
            none.kind = -1;
            prefetch(it, none, cur);
        }
        while (ok && it.kind >= 0) {
            const PItem nx = sc.next();
            Pre nxt{};
            if (nx.kind >= 0 && it.kind == 0) prefetch(nx, it, nxt);
            const int sb = gk & 1;
            const float *ws = wsm + (it.ord & 1) * N1P;
            const int32_t kl = cur.kl;
            const int64_t row_off = (int64_t)it.t * K;
            if (it.kind == 0) {
                // ---------------- pass A item ----------------
                if (it.first) {
                    for (int h = et; h < N1P; h += 128)
                        wsm[(it.ord & 1) * N1P + h] = h < P.N1 ? P.w[(int64_t)it.t * P.N1 + h] : 0.f;
                    // zero the records of every 256-key block pair the token names
                    const uint32_t *pw = P.tok_pairs + (int64_t)it.t * P.nkpw;
                    constexpr int rb = kRecBytes;
                    for (int wd = 0; wd < P.nkpw; ++wd) {
                        uint32_t bits = pw[wd];
                        while (bits) {
                            const int kp = wd * 32 + __ffs(bits) - 1;
                            bits &= bits - 1;
                            uint4 *dst = reinterpret_cast<uint4 *>(
                                static_cast<char *>(P.rec) + ((int64_t)it.t * P.S2m + 256 * kp) * rb);
                            for (int i = et; i < 256 * rb / 16; i += 128) dst[i] = make_uint4(0, 0, 0, 0);
                        }
                    }
                    if (!group_sync(&bars->sm_sync, ph, &ctl.abort, P.status)) { ok = false; break; }
                    m_a = -INFINITY;
                    z_a = 0.f;
                }
                if (!wait_bar(&bars->s_full[sb], (gk >> 1) & 1, &ctl.abort, P.status)) { ok = false; break; }
                tc_fence_after();
                float I2[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t sa = tm_s + (2 * sb + h) * N1P + lane_addr;
                    float sv[32];
                    float I = 0.f;
#pragma unroll 1
                    for (int c = 0; c < N1P; c += kC) {
                        if (kC == 32) tmem_ld32(sa + c, sv); else tmem_ld16(sa + c, sv);
                        float wv[32];
#pragma unroll
                        for (int hh = 0; hh < kC; hh += 4) {
                            const float4 w4 = *reinterpret_cast<const float4 *>(ws + c + hh);
                            wv[hh] = w4.x; wv[hh + 1] = w4.y; wv[hh + 2] = w4.z; wv[hh + 3] = w4.w;
                        }
                        tmem_wait_ld();
                        float i4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int hh = 0; hh < kC; ++hh) i4[hh & 3] = fmaf(wv[hh], fmaxf(sv[hh], 0.f), i4[hh & 3]);
                        I += (i4[0] + i4[1]) + (i4[2] + i4[3]);
                    }
                    I2[h] = I;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->s_empty[sb]);
                float park[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int32_t v = cur.v[h];
                    const bool valid = v >= 0 && v < kl;
                    const float I = I2[h];
                    if (valid) {
                        if (I > m_a) {
                            z_a = (m_a == -INFINITY) ? 0.f : z_a * __expf(m_a - I);
                            m_a = I;
                        }
                        z_a += __expf(I - m_a);
                    }
                    park[h] = valid ? I : -INFINITY;
                    const int j = it.pair * 256 + h * 128 + lrow;
                    if (!kTP && j < K) P.y[row_off + j] = park[h];            // parked for pass B
                }
                if constexpr (kTP) {
                    // parked for pass B in this thread's lane: columns 2 pair, 2 pair + 1 of
                    // the token ordinal's half of the region
                    const uint32_t pa = tmem + kColPark + (it.ord & 1) * 32 + 2 * it.pair + lane_addr;
                    tmem_st2(pa, park[0], park[1]);
                    tmem_st2(pa + 64, __int_as_float(cur.v[0]), __int_as_float(cur.v[1]));
                    tmem_wait_st();
                }
                if (it.last) {
                    float mw = m_a;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) mw = fmaxf(mw, __shfl_xor_sync(0xffffffffu, mw, o));
                    if (lane == 0) ctl.stat_m[ew] = mw;
                    if (!group_sync(&bars->sm_sync, ph, &ctl.abort, P.status)) { ok = false; break; }
                    float M = -INFINITY;
#pragma unroll
                    for (int i = 0; i < 4; ++i) M = fmaxf(M, ctl.stat_m[i]);
                    float zw = (m_a == -INFINITY) ? 0.f : z_a * __expf(m_a - M);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) zw += __shfl_xor_sync(0xffffffffu, zw, o);
                    if (lane == 0) ctl.stat_z[ew] = zw;
                    if (!group_sync(&bars->sm_sync, ph, &ctl.abort, P.status)) { ok = false; break; }
                    float Z = 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) Z += ctl.stat_z[i];
                    M_n = M;
                    iZ_n = Z > 0.f ? 1.f / Z : 0.f;
                }
            } else {
                // ---------------- pass B item ----------------
                if (it.first) {
                    M_b = M_n;
                    iZ_b = iZ_n;
                }
                float dI2[2], y2[2];
                bool valid2[2];
                float Ip[2] = {0.f, 0.f};
                int32_t vb[2] = {cur.v[0], cur.v[1]};
                if constexpr (kTP) {
                    const uint32_t pa = tmem + kColPark + (it.ord & 1) * 32 + 2 * it.pair + lane_addr;
                    float f0, f1;
                    tmem_ld2(pa, Ip[0], Ip[1]);
                    tmem_ld2(pa + 64, f0, f1);
                    tmem_wait_ld();
                    vb[0] = __float_as_int(f0);
                    vb[1] = __float_as_int(f1);
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int j = it.pair * 256 + h * 128 + lrow;
                    const int32_t v = vb[h];
                    valid2[h] = v >= 0 && v < kl;
                    dI2[h] = 0.f;
                    y2[h] = 0.f;
                    if (j < K) {
                        const float I = kTP ? Ip[h] : (cur.haveI ? cur.I[h] : P.y[row_off + j]);
                        y2[h] = valid2[h] ? __expf(I - M_b) * iZ_b : 0.f;
                        dI2[h] = valid2[h] ? y2[h] - cur.p[h] : 0.f;
                    }
                }
                // the dS tile is free once the dq product of the previous pass-B item read it
                if (!wait_bar(&bars->ds_empty, (gd & 1) ^ 1, &ctl.abort, P.status)) { ok = false; break; }
                if (!wait_bar(&bars->s_full[sb], (gk >> 1) & 1, &ctl.abort, P.status)) { ok = false; break; }
                tc_fence_after();
                uint64_t smask2[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t sa = tm_s + (2 * sb + h) * N1P + lane_addr;
                    const uint32_t dwa = tm_dw + lane_addr;
                    uint8_t *dsrow = ds_tile + h * 16384 + lrow * 128;
                    const float dI = dI2[h];
                    const bool zacc = it.first && h == 0;      // the token's first partials
                    uint64_t smask = 0;
#pragma unroll 1
                    for (int c = 0; c < N1P; c += 16) {
                        float sv[16], acc[16], wv[16];
                        tmem_ld16(sa + c, sv);
                        if (!zacc) tmem_ld16(dwa + c, acc);
#pragma unroll
                        for (int hh = 0; hh < 16; hh += 4) {
                            const float4 w4 = *reinterpret_cast<const float4 *>(ws + c + hh);
                            wv[hh] = w4.x; wv[hh + 1] = w4.y; wv[hh + 2] = w4.z; wv[hh + 3] = w4.w;
                        }
                        tmem_wait_ld();
                        uint32_t m16 = 0, pk[8];
#pragma unroll
                        for (int hh = 0; hh < 16; hh += 2) {
                            const float s0 = sv[hh], s1 = sv[hh + 1];
                            acc[hh] = fmaf(dI, fmaxf(s0, 0.f), zacc ? 0.f : acc[hh]);
                            acc[hh + 1] = fmaf(dI, fmaxf(s1, 0.f), zacc ? 0.f : acc[hh + 1]);
                            pk[hh >> 1] = pack2<T>(s0 > 0.f ? dI * wv[hh] : 0.f, s1 > 0.f ? dI * wv[hh + 1] : 0.f);
                            m16 |= (s0 > 0.f ? 1u : 0u) << hh | (s1 > 0.f ? 2u : 0u) << hh;
                        }
                        const int c8 = c >> 3;
                        *reinterpret_cast<uint4 *>(dsrow + (((c8 ^ lrow) & 7) << 4)) =
                            make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        *reinterpret_cast<uint4 *>(dsrow + ((((c8 + 1) ^ lrow) & 7) << 4)) =
                            make_uint4(pk[4], pk[5], pk[6], pk[7]);
                        smask |= (uint64_t)m16 << c;
                        tmem_st16(dwa + c, acc);
                    }
                    smask2[h] = smask;
                    if (h == 0) tmem_wait_st();                 // half 1 reads these columns
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->s_empty[sb]);
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->ds_full);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    // record of this (token, key): the mask words are the same for every slot
                    // naming the key; dI is added, so repeated slots of a key sum their dI
                    const int32_t v = vb[h];
                    if (valid2[h] && v < P.S2m) {
                        constexpr int rb = kRecBytes;
                        char *rp = static_cast<char *>(P.rec) + ((int64_t)it.t * P.S2m + v) * rb;
                        if (N1P > 32) {
                            *reinterpret_cast<uint2 *>(rp) =
                                make_uint2((uint32_t)smask2[h], (uint32_t)(smask2[h] >> 32));
                        } else {
                            *reinterpret_cast<uint32_t *>(rp) = (uint32_t)smask2[h];
                        }
                        if constexpr (kMode == 2) red_add_di_fixed(rp + rec_di_offset(rb), dI2[h]);
                        else red_add_f32(reinterpret_cast<float *>(rp + rec_di_offset(rb)), dI2[h]);
                    }
                    const int j = it.pair * 256 + h * 128 + lrow;
                    if (j < K) P.y[row_off + j] = y2[h];
                }
                if (nx.kind >= 0) prefetch(nx, it, nxt);
                ++gd;
                if (it.last) {
                    // softmax_out of the token's slot tiles outside its non-empty pairs
                    const uint64_t pmask = pair_mask(P.tok_tiles[it.t]);
                    const int ntiles = (K + 127) / 128;
                    for (int tl = 0; tl < ntiles; ++tl) {
                        if ((pmask >> (tl >> 1)) & 1) continue;
                        const int jz = tl * 128 + et;
                        if (jz < K) P.y[row_off + jz] = 0.f;
                    }
                    // dW: the per-slot partials (both halves), then a butterfly over the lanes
                    // that leaves each lane kV / 32 heads, then the 4 warps in a fixed order
                    constexpr int kV = N1P < 32 ? 32 : N1P;
                    float vv[kV];
#pragma unroll
                    for (int hh = 0; hh < kV; ++hh) vv[hh] = 0.f;
#pragma unroll
                    for (int c = 0; c < N1P; c += 16) tmem_ld16(tm_dw + lane_addr + c, vv + c);
                    tmem_wait_ld();
                    int len = kV;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        const int half = len >> 1;
                        const bool upper = (lane & o) != 0;
#pragma unroll
                        for (int hh = 0; hh < kV / 2; ++hh) {
                            if (hh < half) {
                                const float mine = upper ? vv[hh + half] : vv[hh];
                                const float other = upper ? vv[hh] : vv[hh + half];
                                vv[hh] = mine + __shfl_xor_sync(0xffffffffu, other, o);
                            }
                        }
                        len = half;
                    }
                    int base = 0, span = kV;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        span >>= 1;
                        if (lane & o) base += span;
                    }
                    // scratch buffer ord % 2 (the next write to it comes after the following
                    // token's group sync, which every warp reaches only after its reads below)
                    float *rd = red + (it.ord & 1) * 256;
#pragma unroll
                    for (int hh = 0; hh < kV / 32; ++hh) rd[ew * 64 + base + hh] = vv[hh];
                    if (!group_sync(&bars->sm_sync, ph, &ctl.abort, P.status)) { ok = false; break; }
                    for (int hh = et; hh < P.N1; hh += 128) {
                        float a = 0.f;
                        for (int i = 0; i < 4; ++i) a += rd[i * 64 + hh];
                        P.dw[(int64_t)it.t * P.N1 + hh] = a;
                    }
                    // dq^T readback (lane = d): columns = heads
                    if (!wait_bar(&bars->dq_full, nb & 1, &ctl.abort, P.status)) { ok = false; break; }
                    tc_fence_after();
                    if (quad * 32 < D) {
                        T *dqrow = reinterpret_cast<T *>(P.dq) + (int64_t)it.t * P.N1 * D;
                        float dv[32];
#pragma unroll
                        for (int c0 = 0; c0 < N1P; c0 += kC) {
                            if (kC == 32) tmem_ld32(tm_dq + lane_addr + c0, dv); else tmem_ld16(tm_dq + lane_addr + c0, dv);
                            tmem_wait_ld();
#pragma unroll
                            for (int c = 0; c < kC; ++c) {
                                const int hh = c0 + c;
                                if (hh < P.N1) dqrow[(int64_t)hh * D + lrow] = T(dv[c]);
                            }
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->dq_empty);
                    ++nb;
                }
            }
            ++gk;
            it = nx;
            cur = nxt;
        }
    }

    // ---------------- teardown ----------------
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 3) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kPTmemCols));
    }
}

template <int N1P, int D, typename T>
cudaError_t launch_pair_t(const Params &P, int workers, cudaStream_t s) {
    const PPlan sp = pair_plan<N1P>();
    if (sp.total > 226 * 1024) return cudaErrorInvalidConfiguration;
    // logits parked in TMEM for rows of at most 4096 slots (16 tile pairs)
    auto k = P.K <= 4096
                 ? (P.deterministic ? fused_pair_sm100<N1P, D, T, 2, true> : fused_pair_sm100<N1P, D, T, 1, true>)
                 : (P.deterministic ? fused_pair_sm100<N1P, D, T, 2, false> : fused_pair_sm100<N1P, D, T, 1, false>);
    CUtensorMap qmap;
    cudaError_t e = encode_q_map<N1P, T>(P, &qmap);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total);
    if (e != cudaSuccess) return e;
    k<<<workers, kPThreads, sp.total, s>>>(P, qmap);
    return cudaGetLastError();
}

template <int N1P, int D>
cudaError_t launch_pair_d(const Params &P, int workers, cudaStream_t s) {
    return P.dtype == SLIKL_BF16 ? launch_pair_t<N1P, D, __nv_bfloat16>(P, workers, s)
                                 : launch_pair_t<N1P, D, __half>(P, workers, s);
}

template <int N1P>
cudaError_t launch_pair_n(const Params &P, int workers, cudaStream_t s) {
    return P.D == 128 ? launch_pair_d<N1P, 128>(P, workers, s) : launch_pair_d<N1P, 64>(P, workers, s);
}

}  // namespace

// Record mode (key-major dK path) with N1 <= 64, D in {64, 128}, topk <= 8192.
cudaError_t launch_fused_pair_sm100(const Params &P, int workers, cudaStream_t s) {
    if (!P.km || P.N1 > 64 || (P.D != 64 && P.D != 128) || P.K > 64 * 128)
        return cudaErrorInvalidValue;
    if (P.N1 <= 16) return launch_pair_n<16>(P, workers, s);
    if (P.N1 <= 32) return launch_pair_n<32>(P, workers, s);
    return launch_pair_n<64>(P, workers, s);
}

}  // namespace slikl
