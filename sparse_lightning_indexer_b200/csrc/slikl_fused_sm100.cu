// Fused per-token kernel on the sm_100a tensor cores (tcgen05 MMA, accumulators in TMEM).
//
// Per query token t, over its active 128-slot tiles (aclnnSparseLightningIndexerKLLossGrad,
// section "计算公式"):
//   pass A  gather K rows -> smem; S^T[128 keys x N1] = K . q^T          (tcgen05, TMEM)
//           epilogue (one thread per key slot): I = w . ReLU(S) and online max / sum;
//           I is parked in softmax_out.
//   combine m, Z over the token.
//   pass B  gather K rows again; S^T recomputed (tcgen05); epilogue: y = e^(I-m)/Z ->
//           softmax_out, dI = y - p, dW_h += dI ReLU(S_h) (fp32, per thread),
//           dS = dI * w * 1[S > 0] -> bf16/fp16 smem tile [N1 x 128 keys]
//           dq^T[D x N1] += K^T . dS^T                                    (tcgen05, TMEM)
//           dK^T[D x 128 keys] = q^T . dS                                 (tcgen05, TMEM)
//           epilogue: dK^T rows (one thread per d) scatter-added with red.global.add.f32,
//           32 consecutive d per warp instruction (128-byte lines), or stored per slot in
//           deterministic mode.
//   dW reduced over the token in a fixed order; dq^T read back from TMEM.
// Recomputing S in pass B costs a fourth product per tile (8 instead of 6 N1*D*K FLOP per
// token) but keeps the per-thread state to one fp32 accumulator per head; the L2 scatter
// of dK, not the tensor pipe, bounds this kernel.
//
// Warp roles (320 threads): warp 0 gathers (cp.async, 16-byte row chunks, zero-fill for
// invalid slots), warp 1 issues the MMAs (one thread) and owns TMEM, warps 2..9 are two
// epilogue warpgroups that take the tiles of each pass in turn.
//
// Shared-memory tiles use the 128-byte swizzle in 8-row atoms, so one K tile serves as the
// K-major A operand of the S product and as the MN-major A operand of the dq product; the q
// tile is K-major B for S and MN-major A for dK; the dS tile [heads x keys] is K-major B for
// dq and MN-major B for dK.
//
// Every wait on an mbarrier is bounded (about one second of SM clock); on expiry the CTA
// sets SLIKL_DEV_WAIT_TIMEOUT, every role stops, in-flight copies and MMAs are drained, TMEM
// is freed and the kernel returns.
#include <type_traits>

#include "slikl_common.cuh"

namespace slikl {
namespace {

constexpr int kThreads = 320;
constexpr int kEpiThreads = 256;
constexpr long long kWaitCycles = 1ll << 31;
constexpr int kTmemCols = 512;
constexpr int kStageBytes = 128 * 256;      // 128 key rows x 128 d (two 64-d column blocks)

// ------------------------------------------------------------------------------------------
// PTX wrappers
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
        ::"r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 bit, 16 / 32 consecutive columns per thread
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    tmem_ld16(taddr, v);
    tmem_ld16(taddr + 16, v + 16);
}

// Shared-memory matrix descriptor (sm_100): start >> 4 in [0,14), leading byte offset >> 4
// in [16,30), stride byte offset >> 4 in [32,46), version 1 at bit 46, 128-byte swizzle
// (value 2) in [61,64).
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16 with fp32 accumulate: D format bit 4, A/B format at
// bits 7 / 10 (0 = f16, 1 = bf16), A / B MN-major at bits 15 / 16, N >> 3 at 17, M >> 4 at 24.
__host__ __device__ constexpr uint32_t idesc_f16(int fmt, int m, int n, int a_mn, int b_mn) {
    return (1u << 4) | ((uint32_t)fmt << 7) | ((uint32_t)fmt << 10) | ((uint32_t)a_mn << 15) |
           ((uint32_t)b_mn << 16) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// Byte offset of element (row, col) of a tile of 128-byte rows (64 bf16 per row) in 8-row
// atoms with the 128-byte swizzle (16-byte chunk index XOR row % 8).
__device__ __forceinline__ uint32_t sw128(int row, int col_elem) {
    return (uint32_t)(row * 128 + ((((col_elem >> 3) ^ row) & 7) << 4) + (col_elem & 7) * 2);
}

struct Barriers {
    uint64_t kv_full[4], kv_empty[4];
    uint64_t q_full[2], q_empty[2];
    uint64_t s_full[2], s_empty[2];
    uint64_t ds_full[2], ds_empty[2];
    uint64_t dk_full[2], dk_empty[2];
    uint64_t dq_full, dq_empty;
    uint64_t drain;
    uint64_t epi;        // all 8 epilogue warps (reusable barrier)
    uint64_t wgb[2];     // the 4 warps of one epilogue warpgroup
};

struct SmemPlan {
    uint32_t stages, kv, q, ds, w, rows, red, bar, total;
};

template <int N1P>
__host__ __device__ inline SmemPlan plan_smem(int K, int stages) {
    SmemPlan s{};
    uint32_t off = 0;
    auto take = [&](uint32_t bytes, uint32_t align) {
        off = (off + align - 1) / align * align;
        uint32_t o = off;
        off += bytes;
        return o;
    };
    (void)K;
    s.stages = stages;
    s.kv = take(stages * kStageBytes, 1024);
    s.q = take(2 * N1P * 256, 1024);                 // two buffers, 2 column blocks each
    s.ds = take(2 * N1P * 256, 1024);                // two buffers [N1P heads x 128 keys]
    s.w = take(N1P * 4, 16);
    s.rows = take(2 * 128 * 4, 16);
    s.red = take(8 * 64 * 4 + 64, 16);
    s.bar = take(sizeof(Barriers) + 16, 8);
    s.total = off + 1024;                            // slack for aligning the dynamic base
    return s;
}

struct Ctl {
    volatile int abort;
    uint32_t tmem_base;
    float stat_m[8], stat_z[8];
};

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, Ctl *ctl,
                                         uint32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    long long start = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (ctl->abort) return false;
        if (clock64() - start > kWaitCycles) {
            ctl->abort = 1;
            set_status(status, SLIKL_DEV_WAIT_TIMEOUT);
            return false;
        }
    }
}

// Reusable barrier over a fixed set of warps (lane 0 of each arrives); bounded like wait_bar,
// so a CTA that aborts never strands warps at a hardware barrier.
__device__ __forceinline__ bool group_sync(uint64_t *bar, uint32_t &phase, Ctl *ctl,
                                           uint32_t *status) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
    const bool ok = wait_bar(bar, phase & 1, ctl, status);
    ++phase;
    return ok;
}

template <typename T>
__device__ __forceinline__ uint16_t to_bits16(float v);
template <>
__device__ __forceinline__ uint16_t to_bits16<__nv_bfloat16>(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}
template <>
__device__ __forceinline__ uint16_t to_bits16<__half>(float v) {
    return __half_as_ushort(__float2half_rn(v));
}

// ------------------------------------------------------------------------------------------
// The kernel
// ------------------------------------------------------------------------------------------
template <int N1P, int D, typename T, int LAG>
__global__ void __launch_bounds__(kThreads, 1) fused_sm100(Params P, int stages) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int K = P.K;
    const SmemPlan SP = plan_smem<N1P>(K, stages);
    Barriers *bars = reinterpret_cast<Barriers *>(smem + SP.bar);
    __shared__ Ctl ctl;
    constexpr int kFmt = std::is_same<T, __nv_bfloat16>::value ? 1 : 0;
    constexpr uint32_t kIdescS = idesc_f16(kFmt, 128, N1P, 0, 0);
    constexpr uint32_t kIdescDq = idesc_f16(kFmt, 128, N1P, 1, 0);
    constexpr uint32_t kIdescDk = idesc_f16(kFmt, 128, 128, 1, 1);
    constexpr int kDChunks = D / 8;          // 16-byte chunks per key row

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = P.meta[kMetaHeader + 2 * blockIdx.x];
    const int t1 = P.meta[kMetaHeader + 2 * blockIdx.x + 1];

    // ---------------- setup ----------------
    if (threadIdx.x == 0) {
        ctl.abort = 0;
        for (int s = 0; s < stages; ++s) {
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->q_full[b], 1);
            mbar_init(&bars->q_empty[b], 1);
            mbar_init(&bars->s_full[b], 1);
            mbar_init(&bars->s_empty[b], 4);
            mbar_init(&bars->ds_full[b], 4);
            mbar_init(&bars->ds_empty[b], 1);
            mbar_init(&bars->dk_full[b], 1);
            mbar_init(&bars->dk_empty[b], 4);
        }
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_empty, 8);
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->epi, 8);
        mbar_init(&bars->wgb[0], 4);
        mbar_init(&bars->wgb[1], 4);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
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
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&ctl.tmem_base)), "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    const uint32_t tm_s = tmem;              // S^T buffers: columns [0, 2*N1P)
    const uint32_t tm_dq = tmem + 128;       // dq^T: columns [128, 128 + N1P)
    const uint32_t tm_dk = tmem + 256;       // dK^T buffers: columns [256, 512)

    if (warp == 0) {
        // =============================== producer ===============================
        uint64_t *pend[LAG + 1];
        int npend = 0;
        uint32_t gk = 0, tq = 0;
        const char *kbase_ptr = static_cast<const char *>(P.k);
        const int rsub = lane / kDChunks;                 // row within a group of rows
        const int chunk = lane % kDChunks;
        constexpr int kRowsPerPass = 32 / kDChunks;       // 2 (D=128) or 4 (D=64)
        auto signal_done = [&](bool all) {
            if (all) cp_async_wait<0>(); else cp_async_wait<LAG>();
            fence_proxy_async();
            __syncwarp();
            int n = all ? npend : npend - LAG;
            if (lane == 0)
                for (int i = 0; i < n; ++i) mbar_arrive(pend[i]);
            for (int i = 0; i + n < npend; ++i) pend[i] = pend[i + n];
            npend -= n;
        };
        auto push = [&](uint64_t *bar) {
            cp_async_commit();
            pend[npend++] = bar;
            if (npend > LAG) signal_done(false);
        };
        bool ok = true;
        for (int t = t0; t < t1 && ok; ++t) {
            const uint64_t mask = P.tok_tiles[t];
            if (!mask) continue;
            const int32_t kb = P.tok_kbase[t], kl = P.tok_klen[t];
            const int32_t *irow = P.idx + (int64_t)t * K;
            // q tile (rows h < N1) into q buffer tq % 2
            const int qb = tq & 1;
            if (!wait_bar(&bars->q_empty[qb], ((tq >> 1) & 1) ^ 1, &ctl, P.status)) { ok = false; break; }
            {
                const char *qsrc = static_cast<const char *>(P.q) + (int64_t)t * P.N1 * D * 2;
                const uint32_t qdst = smem_u32(smem + SP.q + qb * N1P * 256);
                for (int h = rsub; h < P.N1; h += kRowsPerPass) {
                    const int cb = chunk >> 3;
                    cp_async16(qdst + cb * (N1P * 128) + sw128(h, (chunk & 7) * 8),
                               qsrc + (int64_t)h * D * 2 + chunk * 16, 16);
                }
                push(&bars->q_full[qb]);
            }
            // pass A then pass B: the same gather twice
            for (int pass = 0; pass < 2 && ok; ++pass) {
                uint64_t m = mask;
                while (m) {
                    const int tile = __ffsll((long long)m) - 1;
                    m &= m - 1;
                    const int s = gk % stages;
                    if (!wait_bar(&bars->kv_empty[s], ((gk / stages) & 1) ^ 1, &ctl, P.status)) { ok = false; break; }
                    const uint32_t dst = smem_u32(smem + SP.kv + s * kStageBytes);
                    for (int r = rsub; r < 128; r += kRowsPerPass) {
                        const int j = tile * 128 + r;
                        const int32_t v = j < K ? __ldg(irow + j) : -1;
                        const bool valid = v >= 0 && v < kl;
                        const char *src = kbase_ptr + (valid ? ((int64_t)(kb + v) * D * 2 + chunk * 16) : 0);
                        const int cb = chunk >> 3;
                        cp_async16(dst + cb * 16384 + sw128(r, (chunk & 7) * 8), src, valid ? 16 : 0);
                    }
                    push(&bars->kv_full[s]);
                    ++gk;
                }
            }
            ++tq;
        }
        signal_done(true);
    } else if (warp == 1) {
        // =============================== MMA issuer ===============================
        uint32_t gk = 0, ga = 0, gb = 0, tq = 0;
        bool ok = true;
        const uint32_t kv0 = smem_u32(smem + SP.kv);
        const uint32_t q0 = smem_u32(smem + SP.q);
        const uint32_t ds0 = smem_u32(smem + SP.ds);
        // S^T[128 keys x N1P] = K_tile . q^T into S buffer ga & 1; returns the K stage used
        auto issue_s = [&](uint32_t qaddr, int &stage) -> bool {
            const int s = gk % stages, b = ga & 1;
            if (!wait_bar(&bars->kv_full[s], (gk / stages) & 1, &ctl, P.status)) return false;
            if (!wait_bar(&bars->s_empty[b], ((ga >> 1) & 1) ^ 1, &ctl, P.status)) return false;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t kaddr = kv0 + s * kStageBytes;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    const uint32_t qoff = (ks >> 2) * (N1P * 128) + (ks & 3) * 32;
                    umma_f16(tm_s + b * N1P, sdesc(kaddr + off, 16, 1024),
                             sdesc(qaddr + qoff, 16, 1024), kIdescS, ks > 0);
                }
                umma_commit(&bars->s_full[b]);
            }
            __syncwarp();
            stage = s;
            ++gk; ++ga;
            return true;
        };
        for (int t = t0; t < t1 && ok; ++t) {
            const uint64_t mask = P.tok_tiles[t];
            if (!mask) continue;
            const int ntile = __popcll(mask);
            const int qb = tq & 1;
            const uint32_t qaddr = q0 + qb * N1P * 256;
            if (!wait_bar(&bars->q_full[qb], (tq >> 1) & 1, &ctl, P.status)) { ok = false; break; }
            // ---- pass A: S only; the stage is free once the product is done ----
            for (int i = 0; i < ntile && ok; ++i) {
                int st;
                if (!issue_s(qaddr, st)) { ok = false; break; }
                if (lane == 0) umma_commit(&bars->kv_empty[st]);
                __syncwarp();
            }
            if (!ok) break;
            // ---- pass B: S again (one tile ahead), dq^T += K^T . dS^T, dK^T = q^T . dS ----
            if (!wait_bar(&bars->dq_empty, (tq & 1) ^ 1, &ctl, P.status)) { ok = false; break; }
            int st_cur = 0, st_next = 0;
            if (!issue_s(qaddr, st_cur)) { ok = false; break; }
            for (int i = 0; i < ntile; ++i) {
                if (i + 1 < ntile && !issue_s(qaddr, st_next)) { ok = false; break; }
                const int b = gb & 1;
                if (!wait_bar(&bars->ds_full[b], (gb >> 1) & 1, &ctl, P.status)) { ok = false; break; }
                if (!wait_bar(&bars->dk_empty[b], ((gb >> 1) & 1) ^ 1, &ctl, P.status)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t kaddr = kv0 + st_cur * kStageBytes;
                    const uint32_t dsaddr = ds0 + b * N1P * 256;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {        // 128 keys, 16 per step
                        const uint64_t a = sdesc(kaddr + ks * 2048, 16384, 1024);
                        const uint64_t bd = sdesc(dsaddr + (ks >> 2) * (N1P * 128) + (ks & 3) * 32, 16, 1024);
                        umma_f16(tm_dq, a, bd, kIdescDq, (i > 0 || ks > 0) ? 1u : 0u);
                    }
                    umma_commit(&bars->kv_empty[st_cur]);
#pragma unroll
                    for (int ks = 0; ks < N1P / 16; ++ks) {  // N1P heads, 16 per step
                        const uint64_t a = sdesc(qaddr + ks * 2048, N1P * 128, 1024);
                        const uint64_t bd = sdesc(dsaddr + ks * 2048, N1P * 128, 1024);
                        umma_f16(tm_dk + b * 128, a, bd, kIdescDk, ks > 0);
                    }
                    umma_commit(&bars->dk_full[b]);
                    umma_commit(&bars->ds_empty[b]);
                }
                __syncwarp();
                st_cur = st_next;
                ++gb;
            }
            if (!ok) break;
            if (lane == 0) {
                umma_commit(&bars->dq_full);
                umma_commit(&bars->q_empty[qb]);
            }
            __syncwarp();
            ++tq;
        }
        // drain: wait for every MMA issued by this thread before TMEM is released
        if (lane == 0) umma_commit(&bars->drain);
        __syncwarp();
        {
            long long start = clock64();
            while (!mbar_try_wait(&bars->drain, 0) && clock64() - start < kWaitCycles) {}
        }
    } else {
        // =============================== epilogue ===============================
        const int ew = warp - 2;                 // 0..7
        const int wg = ew >> 2;                  // warpgroup 0 / 1
        const int quad = warp & 3;               // TMEM lane quadrant of this warp
        const int lrow = quad * 32 + lane;       // key slot in tile (pass A/B) or d (scatter)
        const int et = threadIdx.x - 64;         // 0..255
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        float *ws = reinterpret_cast<float *>(smem + SP.w);
        int32_t *rows_s = reinterpret_cast<int32_t *>(smem + SP.rows);
        float *red = reinterpret_cast<float *>(smem + SP.red);
        uint8_t *ds_tiles = smem + SP.ds;
        uint32_t ga = 0, gb = 0, tq = 0, ph_epi = 0, ph_wg = 0;
        bool ok = true;
        constexpr int kC = N1P < 32 ? N1P : 32;  // S columns per TMEM load
        for (int t = t0; t < t1 && ok; ++t) {
            const uint64_t mask = P.tok_tiles[t];
            const int32_t kl = P.tok_klen[t], kbs = P.tok_kbase[t];
            const int32_t *irow = P.idx + (int64_t)t * K;
            const float *prow = P.p + (int64_t)t * K;
            float *yrow = P.y + (int64_t)t * K;
            if (!mask) {
                for (int j = et; j < K; j += kEpiThreads) yrow[j] = 0.f;
                for (int e = et; e < P.N1 * D; e += kEpiThreads)
                    reinterpret_cast<T *>(P.dq)[(int64_t)t * P.N1 * D + e] = T(0.f);
                for (int h = et; h < P.N1; h += kEpiThreads) P.dw[(int64_t)t * P.N1 + h] = 0.f;
                continue;
            }
            // previous token done with ws / red, then w_t in place
            if (!group_sync(&bars->epi, ph_epi, &ctl, P.status)) { ok = false; break; }
            for (int h = et; h < N1P; h += kEpiThreads) ws[h] = h < P.N1 ? P.w[(int64_t)t * P.N1 + h] : 0.f;
            if (!group_sync(&bars->epi, ph_epi, &ctl, P.status)) { ok = false; break; }

            // ---------------- pass A: I = w . ReLU(S), online max / sum ----------------
            float m_t = -INFINITY, z_t = 0.f;
            uint64_t mm = mask;
            while (mm) {
                const int tile = __ffsll((long long)mm) - 1;
                mm &= mm - 1;
                if ((ga & 1) == (uint32_t)wg) {
                    const int sb = ga & 1;
                    const int j = tile * 128 + lrow;
                    const int32_t v = j < K ? irow[j] : -1;
                    const bool valid = v >= 0 && v < kl;
                    if (v != -1 && !valid) set_status(P.status, SLIKL_DEV_INDEX_OUT_OF_RANGE);
                    if (!wait_bar(&bars->s_full[sb], (ga >> 1) & 1, &ctl, P.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = tm_s + sb * N1P + lane_addr;
                    float sv[32];
                    float I = 0.f;
#pragma unroll
                    for (int c = 0; c < N1P; c += kC) {
                        if (kC == 32) tmem_ld32(sa + c, sv); else tmem_ld16(sa + c, sv);
                        tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < kC; ++h) I = fmaf(ws[c + h], fmaxf(sv[h], 0.f), I);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->s_empty[sb]);
                    if (valid) {
                        if (I > m_t) {
                            z_t = (m_t == -INFINITY) ? 0.f : z_t * __expf(m_t - I);
                            m_t = I;
                        }
                        z_t += __expf(I - m_t);
                    }
                    if (j < K) yrow[j] = valid ? I : -INFINITY;       // parked for pass B
                }
                ++ga;
            }
            if (!ok) break;

            // ---------------- softmax statistics over the token ----------------
            float mw = m_t;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mw = fmaxf(mw, __shfl_xor_sync(0xffffffffu, mw, o));
            if (lane == 0) ctl.stat_m[ew] = mw;
            if (!group_sync(&bars->epi, ph_epi, &ctl, P.status)) { ok = false; break; }
            float M = -INFINITY;
#pragma unroll
            for (int i = 0; i < 8; ++i) M = fmaxf(M, ctl.stat_m[i]);
            const float zs = (m_t == -INFINITY) ? 0.f : z_t * __expf(m_t - M);
            float zw = zs;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) zw += __shfl_xor_sync(0xffffffffu, zw, o);
            if (lane == 0) ctl.stat_z[ew] = zw;
            if (!group_sync(&bars->epi, ph_epi, &ctl, P.status)) { ok = false; break; }
            float Z = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) Z += ctl.stat_z[i];
            const float invZ = Z > 0.f ? 1.f / Z : 0.f;

            // ---------------- pass B: y, dI, dS, dW; dK scatter ----------------
            float dW[N1P];
#pragma unroll
            for (int h = 0; h < N1P; ++h) dW[h] = 0.f;
            mm = mask;
            while (mm) {
                const int tile = __ffsll((long long)mm) - 1;
                mm &= mm - 1;
                if ((gb & 1) == (uint32_t)wg) {
                    const int b = wg;
                    const int sb = ga & 1;
                    const int j = tile * 128 + lrow;
                    const int32_t v = j < K ? irow[j] : -1;
                    const bool valid = v >= 0 && v < kl;
                    float dI = 0.f;
                    if (j < K) {
                        const float I = yrow[j];
                        const float y = valid ? __expf(I - M) * invZ : 0.f;
                        yrow[j] = y;
                        dI = valid ? y - prow[j] : 0.f;
                    }
                    if (!wait_bar(&bars->ds_empty[b], ((gb >> 1) & 1) ^ 1, &ctl, P.status)) { ok = false; break; }
                    if (!wait_bar(&bars->s_full[sb], (ga >> 1) & 1, &ctl, P.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = tm_s + sb * N1P + lane_addr;
                    uint8_t *dsb = ds_tiles + b * N1P * 256 + (lrow >> 6) * (N1P * 128);
                    const int jj = lrow & 63;
                    float sv[32];
#pragma unroll
                    for (int c = 0; c < N1P; c += kC) {
                        if (kC == 32) tmem_ld32(sa + c, sv); else tmem_ld16(sa + c, sv);
                        tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < kC; ++h) {
                            const float sval = sv[h];
                            dW[c + h] = fmaf(dI, fmaxf(sval, 0.f), dW[c + h]);
                            const float d = sval > 0.f ? dI * ws[c + h] : 0.f;
                            *reinterpret_cast<uint16_t *>(dsb + sw128(c + h, jj)) = to_bits16<T>(d);
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->s_empty[sb]);
                    rows_s[b * 128 + lrow] = valid ? kbs + v : -1;
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->ds_full[b]);
                    // rows_s of this tile visible to the whole group
                    if (!group_sync(&bars->wgb[wg], ph_wg, &ctl, P.status)) { ok = false; break; }
                    if (!wait_bar(&bars->dk_full[b], (gb >> 1) & 1, &ctl, P.status)) { ok = false; break; }
                    tc_fence_after();
                    if (quad * 32 < D) {
                        const uint32_t da = tm_dk + b * 128 + lane_addr;
                        const int d = lrow;
                        float dv[32];
#pragma unroll 1
                        for (int c0 = 0; c0 < 128; c0 += 32) {
                            tmem_ld32(da + c0, dv);
                            tmem_wait_ld();
#pragma unroll
                            for (int c = 0; c < 32; ++c) {
                                const int32_t r = rows_s[b * 128 + c0 + c];
                                if (r >= 0) {
                                    if (P.deterministic)
                                        P.partials[((int64_t)t * K + tile * 128 + c0 + c) * D + d] = dv[c];
                                    else
                                        red_add_f32(P.dk_acc + (int64_t)r * D + d, dv[c]);
                                }
                            }
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->dk_empty[b]);
                    // rows_s reads done before its next write
                    if (!group_sync(&bars->wgb[wg], ph_wg, &ctl, P.status)) { ok = false; break; }
                }
                ++gb;
                ++ga;
            }
            if (!ok) break;
            // slots of inactive tiles: softmax_out = 0
            {
                const int ntiles = (K + 127) / 128;
                for (int tile = 0; tile < ntiles; ++tile) {
                    if ((mask >> tile) & 1) continue;
                    for (int j = tile * 128 + et; j < (tile + 1) * 128 && j < K; j += kEpiThreads) yrow[j] = 0.f;
                }
            }
            // ---------------- dW: fixed-order reduction over the 256 threads ----------------
            // butterfly reduce-scatter within the warp, then the 8 warps in index order
            {
                constexpr int kV = N1P < 32 ? 32 : N1P;
                float vv[kV];
#pragma unroll
                for (int h = 0; h < kV; ++h) vv[h] = h < N1P ? dW[h] : 0.f;
                int len = kV;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const int half = len >> 1;
                    const bool upper = (lane & o) != 0;
#pragma unroll
                    for (int h = 0; h < kV / 2; ++h) {
                        if (h < half) {
                            const float mine = upper ? vv[h + half] : vv[h];
                            const float other = upper ? vv[h] : vv[h + half];
                            vv[h] = mine + __shfl_xor_sync(0xffffffffu, other, o);
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
#pragma unroll
                for (int h = 0; h < kV / 32; ++h) red[ew * 64 + base + h] = vv[h];
            }
            if (!group_sync(&bars->epi, ph_epi, &ctl, P.status)) { ok = false; break; }
            for (int h = et; h < P.N1; h += kEpiThreads) {
                float a = 0.f;
                for (int i = 0; i < 8; ++i) a += red[i * 64 + h];
                P.dw[(int64_t)t * P.N1 + h] = a;
            }
            // ---------------- dq^T readback ----------------
            if (!wait_bar(&bars->dq_full, tq & 1, &ctl, P.status)) { ok = false; break; }
            tc_fence_after();
            if (quad * 32 < D) {
                constexpr int kHalf = N1P / 2;               // heads read by this warpgroup
                const uint32_t qa = tm_dq + wg * kHalf + lane_addr;
                float dv[32];
                const int d = lrow;
                T *dqrow = reinterpret_cast<T *>(P.dq) + (int64_t)t * P.N1 * D;
                if (kHalf >= 32) tmem_ld32(qa, dv); else tmem_ld16(qa, dv);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < (kHalf < 32 ? kHalf : 32); ++c) {
                    const int h = wg * kHalf + c;
                    if (h < P.N1) dqrow[(int64_t)h * D + d] = T(dv[c]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->dq_empty);
            ++tq;
        }
    }

    // ---------------- teardown ----------------
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols));
    }
}

template <int N1P, int D, typename T>
cudaError_t launch_t(const Params &P, int workers, cudaStream_t s) {
    int stages = 4;
    SmemPlan sp = plan_smem<N1P>(P.K, stages);
    while (sp.total > 226 * 1024 && stages > 2) {
        --stages;
        sp = plan_smem<N1P>(P.K, stages);
    }
    if (sp.total > 226 * 1024) return cudaErrorInvalidConfiguration;
    // The producer signals a gathered tile LAG groups late; in pass B the MMA warp holds two
    // stages (S of tile i+1 is issued before the dq product of tile i), so LAG <= stages - 2
    // keeps the producer from waiting on a stage that only a later signal could free.
    cudaError_t e;
    if (stages == 4) {
        auto k = fused_sm100<N1P, D, T, 2>;
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total);
        if (e != cudaSuccess) return e;
        k<<<workers, kThreads, sp.total, s>>>(P, stages);
    } else if (stages == 3) {
        auto k = fused_sm100<N1P, D, T, 1>;
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total);
        if (e != cudaSuccess) return e;
        k<<<workers, kThreads, sp.total, s>>>(P, stages);
    } else {
        auto k = fused_sm100<N1P, D, T, 0>;
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total);
        if (e != cudaSuccess) return e;
        k<<<workers, kThreads, sp.total, s>>>(P, stages);
    }
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

// Shapes this kernel covers: N1 <= 64 (padded to 16/32/64 heads), D in {64, 128},
// topk <= 8192 (at most 64 tiles). Everything else goes to the CUDA-core kernel.
cudaError_t launch_fused_sm100(const Params &P, int workers, cudaStream_t s, bool *handled) {
    *handled = false;
    if (P.N1 > 64 || (P.D != 64 && P.D != 128) || P.K > 64 * 128) return cudaSuccess;
    *handled = true;
    if (P.N1 <= 16) return launch_n<16>(P, workers, s);
    if (P.N1 <= 32) return launch_n<32>(P, workers, s);
    return launch_n<64>(P, workers, s);
}

}  // namespace slikl
