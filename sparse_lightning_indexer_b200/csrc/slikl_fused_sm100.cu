// Fused per-token kernel on the sm_100a tensor cores (tcgen05 MMA, accumulators in TMEM).
//
// For each query token t of the CTA's range and each of its active 128-slot tiles
// (aclnnSparseLightningIndexerKLLossGrad, section "计算公式"):
//   pass A  K rows of the tile gathered to smem; S^T[128 keys x N1] = K . q^T (tcgen05);
//           I = w . ReLU(S) per slot, online max / sum; I parked in softmax_out.
//   after the last pass-A tile: max and sum combined over the token.
//   pass B  K rows gathered again; S^T recomputed; y = e^(I-m)/Z -> softmax_out, dI = y - p,
//           dW_h += dI ReLU(S_h) (fp32), dS = dI * w * 1[S > 0] -> bf16/fp16 smem tile;
//           dq^T[D x heads] += K^T . dS^T (tcgen05), and then one of
//           - scatter mode: dK^T[D x 128 keys] = q^T . dS (tcgen05), scattered into the fp32
//             key rows with red.global.add.f32, 32 consecutive d per warp instruction (one
//             128-byte line), or stored per slot (deterministic mode);
//           - record mode: a record per named (token, key) - the heads with S > 0 and dI
//             (fp32, or 64-bit fixed point in deterministic mode) - for the key-major dK
//             kernel, after zero-filling the token's named 256-key block pairs during pass A.
//   after the last pass-B tile: dW reduced in a fixed order, dq^T read back from TMEM.
//
// Schedule. All roles walk one deterministic item sequence in which pass A of the CTA's next
// token alternates with pass B of the current one (phase k = B(t_{k-1}) interleaved with
// A(t_k)). Every item gathers one K tile and computes one S tile.
//
// Warp roles (384 threads):
//   warps 0-2   producers: each gathers its share of the rows of every tile with cp.async
//               (16-byte chunks of the 256-byte key rows, zero-fill for invalid slots);
//               warp 0 also loads q by TMA. In record mode warps 4-7 are producers too.
//   warp 3      MMA issuer (one thread) and TMEM owner; the S product runs one item ahead.
//   warps 4-7   scatter group (scatter mode): dK^T tiles from TMEM to the fp32 key rows.
//   warps 8-11  softmax group: pass-A and pass-B epilogues, records, dW, dq readback.
// The 4-warp groups each cover the four TMEM lane quadrants (warp id % 4).
//
// Shared-memory tiles use the 128-byte swizzle in 8-row atoms: the K tile is the K-major A
// operand of the S product and the MN-major A operand of the dq product; the q tile is
// K-major B for S and MN-major A for dK; the dS tile [keys x heads] is MN-major B for dq and
// K-major B for dK.
//
// Every wait on an mbarrier is bounded (about one second of SM clock); on expiry the CTA
// sets SLIKL_DEV_WAIT_TIMEOUT, every role stops, in-flight copies and MMAs are drained, TMEM
// is freed and the kernel returns.
#include <type_traits>

#include "slikl_sm100.cuh"

namespace slikl {
namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr int kTmemCols = 512;
constexpr int kStageBytes = 128 * 256;      // 128 key rows x 128 d (two 64-d column blocks)

struct Barriers {
    uint64_t kv_full[4], kv_empty[4];     // K stages: producers -> MMA -> producers
    uint64_t q_full[2], q_empty[2];       // q tiles: producer 0 -> MMA -> producer 0
    uint64_t s_full[2], s_empty[2];       // S^T in TMEM: MMA -> softmax group -> MMA
    uint64_t ds_full[2];                  // dS tile in smem: softmax group -> MMA
    uint64_t rows_full[2];                // key rows of a dS tile: softmax -> scatter group
    uint64_t dk_full[2], dk_empty[2];     // dK^T in TMEM: MMA -> scatter group -> MMA/softmax
    uint64_t dq_full, dq_empty;           // dq^T in TMEM: MMA -> softmax group -> MMA
    uint64_t drain;
    uint64_t sm_sync;                     // the 4 softmax warps (reusable barrier)
};

struct SmemPlan {
    uint32_t stages, kv, q, ds, w, rows, red, ring, bar, total;
};

// Per producer warp, 4 slots of: 128 slot indices, key base, key count (+ padding).
constexpr int kRingSlot = 136;            // int32 entries per slot
constexpr int kRowsStride = 132;          // int32 entries per key-row buffer (16-byte multiple)

// dS tiles [128 keys x N1P heads] are column blocks of 64 heads (128-byte rows, 16 KB per
// block); with 128 heads there is room for one tile (and one dK^T buffer in TMEM), else two
template <int N1P> __host__ __device__ constexpr int n_ds_tiles() { return N1P > 64 ? 1 : 2; }
template <int N1P> __host__ __device__ constexpr int ds_bytes() { return N1P > 64 ? 32768 : 16384; }
template <int N1P> __host__ __device__ constexpr int red_stride() { return N1P > 64 ? N1P : 64; }
// K stages: four of 32 KB; three with 128 heads (q and dS tiles are twice as large)
template <int N1P> __host__ __device__ constexpr int kv_stages() { return N1P > 64 ? 3 : 4; }

template <int N1P>
__host__ __device__ inline SmemPlan plan_smem(int stages) {
    SmemPlan s{};
    uint32_t off = 0;
    auto take = [&](uint32_t bytes, uint32_t align) {
        off = (off + align - 1) / align * align;
        uint32_t o = off;
        off += bytes;
        return o;
    };
    s.stages = stages;
    s.kv = take(stages * kStageBytes, 1024);
    s.q = take(2 * N1P * 256, 1024);                 // two buffers, 2 column blocks each
    s.ds = take(n_ds_tiles<N1P>() * ds_bytes<N1P>(), 1024);   // dS tiles [128 keys x N1P heads]
    s.w = take(2 * N1P * 4, 16);                     // w of two tokens
    s.rows = take(2 * kRowsStride * 4, 16);          // key rows of the dS tiles
    s.red = take(2 * 4 * red_stride<N1P>() * 4, 16); // dW partials of two tokens
    s.ring = take(7 * 4 * kRingSlot * 4, 16);       // up to 7 producer warps
    s.bar = take(sizeof(Barriers) + 16, 8);
    s.total = off + 1024;                            // slack for aligning the dynamic base
    return s;
}

struct Ctl {
    volatile int abort;
    uint32_t tmem_base;
    float stat_m[4], stat_z[4];
};

// ------------------------------------------------------------------------------------------
// Item schedule shared by every role
// ------------------------------------------------------------------------------------------
struct Item {
    int kind;        // 0 = pass A, 1 = pass B, -1 = none
    int t;           // token row
    int tile;        // 128-slot tile index within the token
    int ord;         // ordinal of the token among the CTA's active tokens
    bool first;      // first tile of this token in this pass
    bool last;       // last tile of this token in this pass
};

// Phase 0 = A(t_0); phase k = B(t_(k-1)) and A(t_k) alternated (B first), then whichever
// remains; the final phase = B(t_last). Tiles of a token are visited in index order. Every
// role runs this for every item, so it stays a handful of instructions per item.
struct Sched {
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
                ma = ma_all = m;
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
    __device__ Item next() {
        Item it;
        it.kind = -1;
        if (!a_on && !b_on) return it;
        const bool take_b = b_on && (!a_on || turn_b);
        turn_b = !turn_b;
        if (take_b) {
            it.kind = 1; it.t = tb; it.ord = ob; it.first = b_first;
            it.tile = __ffsll((long long)mb) - 1;
            mb &= mb - 1;
            it.last = mb == 0;
            b_first = false;
            if (it.last) b_on = false;
        } else {
            it.kind = 0; it.t = ta; it.ord = oa; it.first = a_first;
            it.tile = __ffsll((long long)ma) - 1;
            ma &= ma - 1;
            it.last = ma == 0;
            a_first = false;
            if (it.last) a_on = false;
        }
        if (!a_on && !b_on) {
            // phase ends: its A token becomes the B token of the next phase
            if (a_exists) { tb = ta; ob = oa; mb = ma_all; b_on = true; b_first = true; }
            a_exists = find_a();
            turn_b = true;
        }
        return it;
    }
};

// ------------------------------------------------------------------------------------------
// The kernel
// ------------------------------------------------------------------------------------------
// kMode: 0 = scatter mode; 1 = record mode; 2 = record mode, deterministic (dI in 64-bit
// fixed point, 8-byte records widened to 16)
template <int N1P, int D, typename T, int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    fused_sm100(Params P, int stages, const __grid_constant__ CUtensorMap qmap) {
    constexpr bool kRec = kMode != 0;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int K = P.K;
    const SmemPlan SP = plan_smem<N1P>(stages);
    Barriers *bars = reinterpret_cast<Barriers *>(smem + SP.bar);
    __shared__ Ctl ctl;
    constexpr int kFmt = std::is_same<T, __nv_bfloat16>::value ? 1 : 0;
    constexpr uint32_t kIdescS = idesc_f16(kFmt, 128, N1P, 0, 0);
    // dq^T [D x N1P heads]: dS^T read MN-major from the [keys x heads] tile; dK^T [D x 128
    // keys]: the same tile read K-major
    constexpr uint32_t kIdescDq = idesc_f16(kFmt, 128, N1P, 1, 1);
    constexpr uint32_t kIdescDk = idesc_f16(kFmt, 128, 128, 1, 0);
    constexpr int kDChunks = D / 8;          // 16-byte chunks per key row
    constexpr int kC = N1P < 32 ? N1P : 32;  // S columns per TMEM load
    // record: the ReLU mask word(s) (4, 8 or 16 bytes), then dI (fp32, or 64-bit fixed point)
    constexpr int kRecBytes = N1P > 64 ? 32 : (N1P > 32 || kMode == 2 ? 16 : 8);
    // producer warps: 0-2, and in record mode also 4-7 (the scatter group has no work there)
    constexpr int kProd = kRec ? 7 : 3;
    // S^T buffers in TMEM, dS tiles in smem (and dK^T buffers in TMEM, scatter mode)
    constexpr int kNs = (N1P > 64 && !kRec) ? 1 : 2;
    constexpr int kNd = n_ds_tiles<N1P>();
    constexpr uint32_t kDsBytes = ds_bytes<N1P>();
    // TMEM columns: S^T buffers from 0, then dq^T, the per-slot dW partials and the dK^T
    // buffers (up to 64 heads: 0 / 128 / 192 / 256; 128 heads: S^T x kNs, then 128 each)
    constexpr uint32_t kColDq = N1P <= 64 ? 128 : kNs * 128;
    constexpr uint32_t kColDw = N1P <= 64 ? 192 : kColDq + 128;
    constexpr uint32_t kColDk = N1P <= 64 ? 256 : kColDw + 128;
    static_assert(kColDw + N1P <= kTmemCols, "TMEM columns");
    static_assert(kRec || kColDk + kNd * 128 <= kTmemCols, "TMEM columns (dK^T buffers)");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = P.meta[kMetaHeader + 2 * blockIdx.x];
    const int t1 = P.meta[kMetaHeader + 2 * blockIdx.x + 1];

    // ---------------- setup ----------------
    if (threadIdx.x == 0) {
        ctl.abort = 0;
        for (int s = 0; s < stages; ++s) {
            mbar_init(&bars->kv_full[s], 32 * kProd);   // one arrival per producer thread
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->q_full[b], 1);      // producer 0 (expect_tx) + TMA bytes
            mbar_init(&bars->q_empty[b], 1);
            mbar_init(&bars->s_full[b], 1);
            mbar_init(&bars->s_empty[b], 4);
            mbar_init(&bars->ds_full[b], 4);
            mbar_init(&bars->rows_full[b], 4);
            mbar_init(&bars->dk_full[b], 1);
            mbar_init(&bars->dk_empty[b], kRec ? 1 : 4);
        }
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_empty, 4);
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->sm_sync, 4);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // zero the dS tiles once: heads past N1P stay 0
    for (uint32_t i = threadIdx.x; i < kNd * kDsBytes / 16; i += kThreads)
        reinterpret_cast<uint4 *>(smem + SP.ds)[i] = make_uint4(0, 0, 0, 0);
    // zero the q buffers once: padded heads and, for D = 64, the upper column block stay 0;
    // for D = 64 also the upper column block of every K stage (never written by the gather)
    for (uint32_t i = threadIdx.x; i < (uint32_t)(2 * N1P * 256 / 16); i += kThreads)
        reinterpret_cast<uint4 *>(smem + SP.q)[i] = make_uint4(0, 0, 0, 0);
    if (D == 64) {
        for (int s = 0; s < stages; ++s)
            for (uint32_t i = threadIdx.x; i < 16384 / 16; i += kThreads)
                reinterpret_cast<uint4 *>(smem + SP.kv + s * kStageBytes + 16384)[i] =
                    make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async();
    if (warp == 3) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&ctl.tmem_base)), "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    const uint32_t tm_s = tmem;              // S^T buffers: columns [0, kNs * N1P)
    const uint32_t tm_dq = tmem + kColDq;    // dq^T: N1P columns
    const uint32_t tm_dw = tmem + kColDw;    // per-slot dW partial sums: N1P columns
    const uint32_t tm_dk = tmem + kColDk;    // dK^T buffers: kNd x 128 columns (scatter mode)
    int32_t *rows_s = reinterpret_cast<int32_t *>(smem + SP.rows);   // [2][kRowsStride]

    Sched sc;
    sc.init(P.tok_tiles, t0, t1);

    if (warp < 3 || (kRec && warp >= 4 && warp < 8)) {
        // =============================== producers ===============================
        // Every producer warp walks every item in order and waits on every stage phase (a warp
        // that skipped items could be fooled by the phase parity of a reused stage); each warp
        // copies its share of the tile's row groups. Every lane ends an item with
        // cp.async.mbarrier.arrive.noinc, so a stage turns full (32 arrivals per producer warp) when all of its
        // copies have landed, without any producer waiting for them (that arrival also waits
        // for every earlier cp.async of the thread, so nothing else is copied with cp.async).
        // The slot indices, key base and key count of an item are loaded into registers four
        // items ahead and stored into a 4-slot ring in shared memory two items ahead; warp 0
        // also loads q by TMA.
        const int rsub = lane / kDChunks;                 // row within a group of rows
        const int chunk = lane % kDChunks;
        constexpr int kRowsPerPass = 32 / kDChunks;       // 2 (D=128) or 4 (D=64)
        const char *kbase_ptr = static_cast<const char *>(P.k);
        const int pw = warp < 3 ? warp : warp - 1;      // producer index 0 .. kProd - 1
        int32_t *ring = reinterpret_cast<int32_t *>(smem + SP.ring) + pw * 4 * kRingSlot;
        bool ok = true;
        auto arrive_on_copies = [&](uint64_t *bar) {
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
                         : "memory");
        };
        struct IdxRegs { int32_t v[4]; int32_t kb, kl; };
        // lane l loads slots l, l+32, l+64, l+96 of the item's tile (-1 past the token's end)
        auto ldg_idx = [&](const Item &it, IdxRegs &r) {
            const int32_t *irow = P.idx + (int64_t)it.t * K;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = it.tile * 128 + lane + 32 * u;
                r.v[u] = j < K ? irow[j] : -1;
            }
            r.kb = P.tok_kbase[it.t];
            r.kl = P.tok_klen[it.t];
        };
        auto sts_idx = [&](const IdxRegs &r, int slot) {
            int32_t *d = ring + slot * kRingSlot;
#pragma unroll
            for (int u = 0; u < 4; ++u) d[lane + 32 * u] = r.v[u];
            if (lane == 0) { d[128] = r.kb; d[129] = r.kl; }
        };
        Item it0 = sc.next();
        Item it1 = it0.kind >= 0 ? sc.next() : it0;
        Item it2 = it1.kind >= 0 ? sc.next() : it1;
        Item it3 = it2.kind >= 0 ? sc.next() : it2;
        IdxRegs r2{}, r3{};
        if (it0.kind >= 0) { IdxRegs r; ldg_idx(it0, r); sts_idx(r, 0); }
        if (it1.kind >= 0) { IdxRegs r; ldg_idx(it1, r); sts_idx(r, 1); }
        if (it2.kind >= 0) ldg_idx(it2, r2);
        if (it3.kind >= 0) ldg_idx(it3, r3);
        int q_last = -1;                                  // ordinal of the last q load issued
        uint32_t g = 0;
        while (ok && it0.kind >= 0) {
            __syncwarp();                                 // ring stores of earlier items
            if (warp == 0 && it0.kind == 0 && it0.first) {
                // q tile of a new token (heads past N1 read as zero) into q buffer ord % 2
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
            const int s = g % stages;
            if (!wait_bar(&bars->kv_empty[s], ((g / stages) & 1) ^ 1, &ctl.abort, P.status)) { ok = false; break; }
            const int32_t *slot = ring + (g & 3) * kRingSlot;
            const int32_t kb = slot[128], kl = slot[129];
            const int jbase = it0.tile * 128;
            const uint32_t dst = smem_u32(smem + SP.kv + s * kStageBytes) + (chunk >> 3) * 16384;
            // this warp's row groups i = pw, pw + kProd, ...: all slot indices into registers
            // first, then the copies back to back (a shared-memory load issued after a copy
            // waits behind it in the memory pipeline)
            constexpr int kGroups = 128 / kRowsPerPass;       // 64 (D=128) or 32 (D=64)
            constexpr int kPer = (kGroups + kProd - 1) / kProd;
            int32_t vv[kPer];
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int i = pw + kProd * j;
                vv[j] = i < kGroups ? slot[rsub + kRowsPerPass * i] : -1;
            }
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int i = pw + kProd * j;
                if (i < kGroups) {
                    const int r = rsub + kRowsPerPass * i;
                    const int32_t v = vv[j];
                    const bool valid = jbase + r < K && v >= 0 && v < kl;
                    const char *src = kbase_ptr + (valid ? ((int64_t)(kb + v) * (D * 2) + chunk * 16) : 0);
                    cp_async16(dst + sw128(r, (chunk & 7) * 8), src, valid ? 16 : 0);
                }
            }
            arrive_on_copies(&bars->kv_full[s]);
            // ring slot of item g + 2 from the loads issued two items ago; loads of item g + 4
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
            // the CTA stops: wait (bounded) for the last q load before the buffer goes away
            const long long st = clock64();
            while (!mbar_try_wait(&bars->q_full[q_last & 1], (q_last >> 1) & 1) &&
                   clock64() - st < kWaitCycles) {}
        }
    } else if (warp == 3) {
        // =============================== MMA issuer ===============================
        uint32_t gk = 0, gd = 0, nb = 0;       // items, pass-B items, finished B tokens
        bool ok = true;
        const uint32_t kv0 = smem_u32(smem + SP.kv);
        const uint32_t q0 = smem_u32(smem + SP.q);
        const uint32_t ds0 = smem_u32(smem + SP.ds);
        // S^T of item gk into S buffer gk % 2 (pass-A stages are released right away)
        auto issue_s = [&](const Item &it, int &stage) -> bool {
            const int s = gk % stages, b = gk % kNs;
            const int qb = it.ord & 1;
            if (it.kind == 0 && it.first &&
                !wait_bar(&bars->q_full[qb], (it.ord >> 1) & 1, &ctl.abort, P.status)) return false;
            if (!wait_bar(&bars->kv_full[s], (gk / stages) & 1, &ctl.abort, P.status)) return false;
            if (!wait_bar(&bars->s_empty[b], ((gk / kNs) & 1) ^ 1, &ctl.abort, P.status)) return false;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t kaddr = kv0 + s * kStageBytes;
                const uint32_t qaddr = q0 + qb * N1P * 256;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    const uint32_t qoff = (ks >> 2) * (N1P * 128) + (ks & 3) * 32;
                    umma_f16(tm_s + b * N1P, sdesc(kaddr + off, 16, 1024),
                             sdesc(qaddr + qoff, 16, 1024), kIdescS, ks > 0);
                }
                umma_commit(&bars->s_full[b]);
                if (it.kind == 0) umma_commit(&bars->kv_empty[s]);
            }
            __syncwarp();
            stage = s;
            ++gk;
            return true;
        };
        Item cur = sc.next();
        int st_cur = 0, st_nxt = 0;
        if (cur.kind >= 0 && !issue_s(cur, st_cur)) ok = false;
        while (ok && cur.kind >= 0) {
            const Item nxt = sc.next();
            if (nxt.kind >= 0 && !issue_s(nxt, st_nxt)) { ok = false; break; }
            if (cur.kind == 1) {
                const int b = gd % kNd;
                if (cur.first && !wait_bar(&bars->dq_empty, (nb & 1) ^ 1, &ctl.abort, P.status)) { ok = false; break; }
                if (!wait_bar(&bars->ds_full[b], (gd / kNd) & 1, &ctl.abort, P.status)) { ok = false; break; }
                if (!kRec && !wait_bar(&bars->dk_empty[b], ((gd / kNd) & 1) ^ 1, &ctl.abort, P.status)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t kaddr = kv0 + st_cur * kStageBytes;
                    const uint32_t dsaddr = ds0 + b * kDsBytes;
                    const uint32_t qaddr = q0 + (cur.ord & 1) * N1P * 256;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {        // 128 keys, 16 per step
                        const uint64_t a = sdesc(kaddr + ks * 2048, 16384, 1024);
                        const uint64_t bd = sdesc(dsaddr + ks * 2048, 16384, 1024);
                        umma_f16(tm_dq, a, bd, kIdescDq, (!cur.first || ks > 0) ? 1u : 0u);
                    }
                    umma_commit(&bars->kv_empty[st_cur]);
                    if constexpr (kRec) {
                        umma_commit(&bars->dk_empty[b]);     // dS tile b read by the dq product
                    } else {
#pragma unroll
                        for (int ks = 0; ks < N1P / 16; ++ks) {  // N1P heads, 16 per step
                            const uint64_t a = sdesc(qaddr + ks * 2048, N1P * 128, 1024);
                            const uint64_t bd = sdesc(dsaddr + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                            umma_f16(tm_dk + b * 128, a, bd, kIdescDk, ks > 0);
                        }
                        umma_commit(&bars->dk_full[b]);
                    }
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
        // drain: wait for every MMA issued by this thread before TMEM is released
        if (lane == 0) umma_commit(&bars->drain);
        __syncwarp();
        {
            long long start = clock64();
            while (!mbar_try_wait(&bars->drain, 0) && clock64() - start < kWaitCycles) {}
        }
    } else if (warp < 8) {
        // =============================== scatter group ===============================
        // (idle when dK is formed key-major from records)
        if constexpr (!kRec) {
        const int quad = warp & 3;
        const int d = quad * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        uint32_t gd = 0;
        bool ok = true;
        while (ok) {
            const Item it = sc.next();
            if (it.kind < 0) break;
            if (it.kind != 1) continue;
            const int b = gd % kNd;
            if (!wait_bar(&bars->rows_full[b], (gd / kNd) & 1, &ctl.abort, P.status)) { ok = false; break; }
            if (!wait_bar(&bars->dk_full[b], (gd / kNd) & 1, &ctl.abort, P.status)) { ok = false; break; }
            tc_fence_after();
            if (quad * 32 < D) {
                // 4 chunks of 32 keys, one compact loop body (the instruction cache of a
                // sub-partition is shared with two other warp roles)
                const int4 *rs4 = reinterpret_cast<const int4 *>(rows_s + b * kRowsStride);
                const int64_t slot0 = (int64_t)it.t * K + it.tile * 128;
                const uint32_t da = tm_dk + b * 128 + lane_addr;
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    float vals[32];
                    tmem_ld32(da + ch * 32, vals);
                    int32_t rr[32];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int4 q4 = rs4[ch * 8 + u];
                        rr[4 * u] = q4.x; rr[4 * u + 1] = q4.y; rr[4 * u + 2] = q4.z; rr[4 * u + 3] = q4.w;
                    }
                    tmem_wait_ld();
                    if (!P.deterministic) {
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            if (rr[c] >= 0) red_add_f32(P.dk_acc + (int64_t)rr[c] * D + d, vals[c]);
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            if (rr[c] >= 0) P.partials[(slot0 + ch * 32 + c) * D + d] = vals[c];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->dk_empty[b]);
            ++gd;
        }
        }
    } else {
        // =============================== softmax group ===============================
        const int ew = warp - 8;                 // 0..3
        const int quad = warp & 3;
        const int lrow = quad * 32 + lane;       // key slot in the tile, or d for dq
        const int et = threadIdx.x - 256;        // 0..127
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        float *wsm = reinterpret_cast<float *>(smem + SP.w);      // [2][N1P]
        float *red = reinterpret_cast<float *>(smem + SP.red);    // [2][4][64]
        uint8_t *ds_tiles = smem + SP.ds;
        uint32_t gk = 0, gd = 0, nb = 0, ph = 0;
        bool ok = true;
        // tokens of the range without any active tile: zero outputs
        for (int t = t0; t < t1; ++t) {
            if (P.tok_tiles[t]) continue;
            for (int j = et; j < K; j += 128) P.y[(int64_t)t * K + j] = 0.f;
            for (int e = et; e < P.N1 * D; e += 128)
                reinterpret_cast<T *>(P.dq)[(int64_t)t * P.N1 * D + e] = T(0.f);
            for (int h = et; h < P.N1; h += 128) P.dw[(int64_t)t * P.N1 + h] = 0.f;
        }
        float m_a = -INFINITY, z_a = 0.f;        // pass-A token: running max / sum
        float M_n = -INFINITY, iZ_n = 0.f;       // its combined statistics, handed to pass B
        float M_b = -INFINITY, iZ_b = 0.f;       // pass-B token
        // per-slot inputs of the next item are loaded while the current one is processed
        struct Pre { int32_t v, kl, kb; float p, I; bool haveI; };
        auto prefetch = [&](const Item &nx, const Item &cu, Pre &o) {
            const int jn = nx.tile * 128 + lrow;
            const int64_t ro = (int64_t)nx.t * K;
            o.kl = P.tok_klen[nx.t];
            o.kb = P.tok_kbase[nx.t];
            o.v = jn < K ? P.idx[ro + jn] : -1;
            o.p = (nx.kind == 1 && jn < K) ? P.p[ro + jn] : 0.f;
            // the parked logit of a pass-B tile is written by the pass-A item of the same
            // tile; when that is the current item it is read later, after it has been parked
            o.haveI = nx.kind == 1 && !(cu.kind == 0 && cu.t == nx.t && cu.tile == nx.tile);
            o.I = (o.haveI && jn < K) ? P.y[ro + jn] : 0.f;
        };
        Item it = sc.next();
        Pre cur{};
        if (it.kind >= 0) {
            Item none;
            none.kind = -1;
            prefetch(it, none, cur);
        }
        while (ok && it.kind >= 0) {
            const Item nx = sc.next();
            Pre nxt{};
            // pass-A items load the next item's inputs right away; pass-B items after their
            // proxy fence (which would otherwise also wait for these loads)
            if (nx.kind >= 0 && it.kind == 0) prefetch(nx, it, nxt);
            const int sb = gk % kNs;
            const float *ws = wsm + (it.ord & 1) * N1P;
            const int32_t kl = cur.kl;
            const int j = it.tile * 128 + lrow;
            const int64_t row_off = (int64_t)it.t * K;
            if (it.kind == 0) {
                // ---------------- pass A item ----------------
                if (it.first) {
                    // w of the new token into its buffer (the token two ordinals back is done)
                    for (int h = et; h < N1P; h += 128)
                        wsm[(it.ord & 1) * N1P + h] = h < P.N1 ? P.w[(int64_t)it.t * P.N1 + h] : 0.f;
                    if constexpr (kRec) {
                        // zero the records of every 256-key block pair the token names; pass B
                        // then adds the named keys (the group syncs that end pass A order
                        // these stores before those)
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
                    }
                    if (!group_sync(&bars->sm_sync, ph, &ctl.abort, P.status)) { ok = false; break; }
                    m_a = -INFINITY;
                    z_a = 0.f;
                }
                const int32_t v = cur.v;
                const bool valid = v >= 0 && v < kl;   // (the metadata pass checked the index)
                if (!wait_bar(&bars->s_full[sb], (gk / kNs) & 1, &ctl.abort, P.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t sa = tm_s + sb * N1P + lane_addr;
                float sv[32];
                float I = 0.f;
#pragma unroll 1
                for (int c = 0; c < N1P; c += kC) {
                    if (kC == 32) tmem_ld32(sa + c, sv); else tmem_ld16(sa + c, sv);
                    float wv[32];
#pragma unroll
                    for (int h = 0; h < kC; h += 4) {
                        const float4 w4 = *reinterpret_cast<const float4 *>(ws + c + h);
                        wv[h] = w4.x; wv[h + 1] = w4.y; wv[h + 2] = w4.z; wv[h + 3] = w4.w;
                    }
                    tmem_wait_ld();
                    float i4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int h = 0; h < kC; ++h) i4[h & 3] = fmaf(wv[h], fmaxf(sv[h], 0.f), i4[h & 3]);
                    I += (i4[0] + i4[1]) + (i4[2] + i4[3]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->s_empty[sb]);
                if (valid) {
                    if (I > m_a) {
                        z_a = (m_a == -INFINITY) ? 0.f : z_a * __expf(m_a - I);
                        m_a = I;
                    }
                    z_a += __expf(I - m_a);
                }
                if (j < K) P.y[row_off + j] = valid ? I : -INFINITY;       // parked for pass B
                if (it.last) {
                    // combine max and sum over the 128 threads (fixed order)
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
                    // stat_m / stat_z are rewritten only after two more group syncs
                }
            } else {
                // ---------------- pass B item ----------------
                if (it.first) {
                    M_b = M_n;
                    iZ_b = iZ_n;
                }
                const int b = gd % kNd;
                const int32_t v = cur.v;
                const bool valid = v >= 0 && v < kl;
                float dI = 0.f, y = 0.f;
                if (j < K) {
                    const float I = cur.haveI ? cur.I : P.y[row_off + j];
                    y = valid ? __expf(I - M_b) * iZ_b : 0.f;
                    dI = valid ? y - cur.p : 0.f;
                }
                // dS tile / key rows of buffer b free once the scatter of its previous use ended
                if (!wait_bar(&bars->dk_empty[b], ((gd / kNd) & 1) ^ 1, &ctl.abort, P.status)) { ok = false; break; }
                if (!wait_bar(&bars->s_full[sb], (gk / kNs) & 1, &ctl.abort, P.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t sa = tm_s + sb * N1P + lane_addr;
                const uint32_t dwa = tm_dw + lane_addr;
                // this slot's row of the [keys x heads] dS tile: 128 bytes per 64-head column
                // block, 16-byte chunks swizzled
                uint8_t *dsrow = ds_tiles + b * kDsBytes + lrow * 128;
                uint64_t smask = 0, smask_hi = 0;   // heads with S > 0 (record mode)
                // 16 heads at a time: dS to smem; this slot's dW partial sums stay in TMEM
#pragma unroll 1
                for (int c = 0; c < N1P; c += 16) {
                    float sv[16], acc[16], wv[16];
                    tmem_ld16(sa + c, sv);
                    if (!it.first) tmem_ld16(dwa + c, acc);
#pragma unroll
                    for (int h = 0; h < 16; h += 4) {
                        const float4 w4 = *reinterpret_cast<const float4 *>(ws + c + h);
                        wv[h] = w4.x; wv[h + 1] = w4.y; wv[h + 2] = w4.z; wv[h + 3] = w4.w;
                    }
                    tmem_wait_ld();
                    uint32_t m16 = 0, pk[8];
#pragma unroll
                    for (int h = 0; h < 16; h += 2) {
                        const float s0 = sv[h], s1 = sv[h + 1];
                        acc[h] = fmaf(dI, fmaxf(s0, 0.f), it.first ? 0.f : acc[h]);
                        acc[h + 1] = fmaf(dI, fmaxf(s1, 0.f), it.first ? 0.f : acc[h + 1]);
                        pk[h >> 1] = pack2<T>(s0 > 0.f ? dI * wv[h] : 0.f, s1 > 0.f ? dI * wv[h + 1] : 0.f);
                        if (kRec) m16 |= (s0 > 0.f ? 1u : 0u) << h | (s1 > 0.f ? 2u : 0u) << h;
                    }
                    const int c8 = (c & 63) >> 3;   // 16-byte chunk of heads c .. c + 7
                    uint8_t *dsblk = dsrow + (c >> 6) * 16384;
                    *reinterpret_cast<uint4 *>(dsblk + (((c8 ^ lrow) & 7) << 4)) =
                        make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    *reinterpret_cast<uint4 *>(dsblk + ((((c8 + 1) ^ lrow) & 7) << 4)) =
                        make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    if (kRec) {
                        if (c < 64) smask |= (uint64_t)m16 << c;
                        else smask_hi |= (uint64_t)m16 << (c - 64);
                    }
                    tmem_st16(dwa + c, acc);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->s_empty[sb]);
                if (!kRec) rows_s[b * kRowsStride + lrow] = valid ? cur.kb + v : -1;
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&bars->ds_full[b]);
                    if (!kRec) mbar_arrive(&bars->rows_full[b]);
                }
                if constexpr (kRec) {
                    // record of this (token, key): the mask words are the same for every slot
                    // naming the key; dI is added, so repeated slots of a key sum their dI
                    if (valid && v < P.S2m) {
                        constexpr int rb = kRecBytes;
                        char *rp = static_cast<char *>(P.rec) + ((int64_t)it.t * P.S2m + v) * rb;
                        if (N1P > 64) {
                            *reinterpret_cast<uint4 *>(rp) =
                                make_uint4((uint32_t)smask, (uint32_t)(smask >> 32),
                                           (uint32_t)smask_hi, (uint32_t)(smask_hi >> 32));
                        } else if (N1P > 32) {
                            *reinterpret_cast<uint2 *>(rp) = make_uint2((uint32_t)smask, (uint32_t)(smask >> 32));
                        } else {
                            *reinterpret_cast<uint32_t *>(rp) = (uint32_t)smask;
                        }
                        if constexpr (kMode == 2) red_add_di_fixed(rp + rec_di_offset(rb), dI);
                        else red_add_f32(reinterpret_cast<float *>(rp + rec_di_offset(rb)), dI);
                    }
                }
                if (j < K) P.y[row_off + j] = y;
                if (nx.kind >= 0) prefetch(nx, it, nxt);
                ++gd;
                if (it.last) {
                    // softmax_out of the token's inactive tiles
                    const uint64_t mask = P.tok_tiles[it.t];
                    const int ntiles = (K + 127) / 128;
                    for (int tl = 0; tl < ntiles; ++tl) {
                        if ((mask >> tl) & 1) continue;
                        for (int jz = tl * 128 + et; jz < (tl + 1) * 128 && jz < K; jz += 128) P.y[row_off + jz] = 0.f;
                    }
                    // per 64-head block (32 columns at least): the 32 lanes' partials summed
                    // by a butterfly that leaves each lane kVW / 32 heads, then the 4 warps
                    // summed in a fixed order through shared memory
                    constexpr int kVW = N1P < 32 ? 32 : (N1P > 64 ? 64 : N1P);
                    constexpr int kRS = red_stride<N1P>();
                    int base = 0, span = kVW;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        span >>= 1;
                        if (lane & o) base += span;
                    }
                    // dW partials in buffer ord % 2: a warp may reach the next token's write
                    // before the others have read this one (nothing in between waits on them);
                    // it writes this buffer again two tokens on, after the next token's group
                    // sync, which every warp reaches only after its reads below
                    float *rd = red + (it.ord & 1) * 4 * kRS;
#pragma unroll
                    for (int hb = 0; hb < N1P; hb += kVW) {
                        float vv[kVW];
#pragma unroll
                        for (int h = 0; h < kVW; ++h) vv[h] = 0.f;
#pragma unroll
                        for (int c = 0; c < kVW && hb + c < N1P; c += 16)
                            tmem_ld16(tm_dw + lane_addr + hb + c, vv + c);
                        tmem_wait_ld();
                        int len = kVW;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) {
                            const int half = len >> 1;
                            const bool upper = (lane & o) != 0;
#pragma unroll
                            for (int h = 0; h < kVW / 2; ++h) {
                                if (h < half) {
                                    const float mine = upper ? vv[h + half] : vv[h];
                                    const float other = upper ? vv[h] : vv[h + half];
                                    vv[h] = mine + __shfl_xor_sync(0xffffffffu, other, o);
                                }
                            }
                            len = half;
                        }
#pragma unroll
                        for (int h = 0; h < kVW / 32; ++h) rd[ew * kRS + hb + base + h] = vv[h];
                    }
                    if (!group_sync(&bars->sm_sync, ph, &ctl.abort, P.status)) { ok = false; break; }
                    for (int h = et; h < P.N1; h += 128) {
                        float a = 0.f;
                        for (int i = 0; i < 4; ++i) a += rd[i * kRS + h];
                        P.dw[(int64_t)it.t * P.N1 + h] = a;
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
                                const int h = c0 + c;
                                if (h < P.N1) dqrow[(int64_t)h * D + lrow] = T(dv[c]);
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
                     "r"(kTmemCols));
    }
}

template <int N1P, int D, typename T>
cudaError_t launch_t(const Params &P, int workers, cudaStream_t s) {
    const int stages = kv_stages<N1P>();
    const SmemPlan sp = plan_smem<N1P>(stages);
    if (sp.total > 226 * 1024) return cudaErrorInvalidConfiguration;
    auto k = !P.km ? fused_sm100<N1P, D, T, 0>
                   : (P.deterministic ? fused_sm100<N1P, D, T, 2> : fused_sm100<N1P, D, T, 1>);
    CUtensorMap qmap;
    cudaError_t e = encode_q_map<N1P, T>(P, &qmap);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total);
    if (e != cudaSuccess) return e;
    k<<<workers, kThreads, sp.total, s>>>(P, stages, qmap);
    return cudaGetLastError();
}

template <int N1P, int D>
cudaError_t launch_d(const Params &P, int workers, cudaStream_t s) {
    return P.dtype == SLIKL_BF16 ? launch_t<N1P, D, __nv_bfloat16>(P, workers, s)
                                 : launch_t<N1P, D, __half>(P, workers, s);
}

template <int N1P>
cudaError_t launch_n(const Params &P, int workers, cudaStream_t s) {
    return P.D == 128 ? launch_d<N1P, 128>(P, workers, s) : launch_d<N1P, 64>(P, workers, s);
}

}  // namespace

// Shapes: N1 <= 128 (padded to 16/32/64/128 heads), D in {64, 128}, topk <= 8192 (at most
// 64 tiles): every problem the entry points accept.
cudaError_t launch_fused_sm100(const Params &P, int workers, cudaStream_t s) {
    if (P.N1 > 128 || (P.D != 64 && P.D != 128) || P.K > 64 * 128) return cudaErrorInvalidValue;
    // record mode up to 64 heads: items of two slot tiles
    if (P.km && P.N1 <= 64) return launch_fused_pair_sm100(P, workers, s);
    if (P.N1 <= 16) return launch_n<16>(P, workers, s);
    if (P.N1 <= 32) return launch_n<32>(P, workers, s);
    if (P.N1 <= 64) return launch_n<64>(P, workers, s);
    return launch_n<128>(P, workers, s);
}

}  // namespace slikl
