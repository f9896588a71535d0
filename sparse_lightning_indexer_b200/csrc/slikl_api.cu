// C ABI of the library (declarations and contract in include/slikl.h).
//
// Two-phase call, after aclnnSparseLightningIndexerKLLossGrad ("函数原型": a first call that
// validates the parameters and returns the workspace size, then the launch on a stream).
// Validation follows the page's constraints ("公共约束" and "规格约束") restricted to what
// this sm_100a build supports.
#include <string.h>

#include "slikl_common.cuh"

namespace slikl {

// per-row KL loss output (slikl_loss.cu)
cudaError_t launch_kl_loss(const Params &P, float *loss, cudaStream_t s);

namespace {

struct Derived {
    int64_t T1, T2;
    KmShape km;
};

slikl_status validate(const slikl_problem *pr, Derived *out) {
    if (!pr) return SLIKL_ERR_PARAM_NULLPTR;
    if (pr->dtype != SLIKL_FP16 && pr->dtype != SLIKL_BF16) return SLIKL_ERR_PARAM_INVALID;
    if (pr->layout_q != SLIKL_BSND && pr->layout_q != SLIKL_TND) return SLIKL_ERR_PARAM_INVALID;
    if (pr->layout_k != SLIKL_BSND && pr->layout_k != SLIKL_TND) return SLIKL_ERR_PARAM_INVALID;
    if (pr->deterministic != 0 && pr->deterministic != 1) return SLIKL_ERR_PARAM_INVALID;
    if (pr->B < 1 || pr->B > (int64_t(1) << 30)) return SLIKL_ERR_PARAM_INVALID;
    if (pr->N1 < 1 || pr->N1 > 128) return SLIKL_ERR_PARAM_INVALID;
    if (pr->D != 64 && pr->D != 128) return SLIKL_ERR_PARAM_INVALID;
    if (pr->topk < 1 || pr->topk > 8192) return SLIKL_ERR_PARAM_INVALID;
    int64_t T1, T2;
    if (pr->layout_q == SLIKL_BSND) {
        if (pr->S1 < 1) return SLIKL_ERR_PARAM_INVALID;
        T1 = pr->B * pr->S1;
    } else {
        if (pr->T1 < 0) return SLIKL_ERR_PARAM_INVALID;
        T1 = pr->T1;
    }
    if (pr->layout_k == SLIKL_BSND) {
        if (pr->S2 < 1) return SLIKL_ERR_PARAM_INVALID;
        T2 = pr->B * pr->S2;
    } else {
        if (pr->T2 < 0) return SLIKL_ERR_PARAM_INVALID;
        T2 = pr->T2;
    }
    if (T1 * pr->topk >= (int64_t(1) << 31) || T2 >= (int64_t(1) << 31) - 2)
        return SLIKL_ERR_PARAM_INVALID;
    out->T1 = T1;
    out->T2 = T2;
    out->km = KmShape{};
    return SLIKL_OK;
}

// Longest key range the key-major path may assume: S2 for BSND keys; for TND keys the
// caller's bound in problem->S2 (0 = none given).
int64_t key_range_bound(const slikl_problem *pr) { return pr->S2 > 0 ? pr->S2 : 0; }

// Whether the key-major dK path can run this problem: a known key-range bound of at most
// 16384 keys.
bool km_possible(const slikl_problem *pr) {
    const int64_t s2 = key_range_bound(pr);
    return s2 > 0 && s2 <= 16384;
}

// Picks the dK path. The key-major path does work in proportion to the (query row, 256-key
// block) pairs that are named at all and the scatter path in proportion to the named slots;
// with the key range at most 16x top-k the first is the cheaper on B200 (measured rates: a
// key-major row of 256 keys costs about as much tensor time as 16 fp32 slot scatters).
slikl_status choose_dk_path(const slikl_problem *pr, Derived *dv, int32_t path) {
    if (path != SLIKL_DK_AUTO && path != SLIKL_DK_SCATTER && path != SLIKL_DK_KEYMAJOR)
        return SLIKL_ERR_PARAM_INVALID;
    const bool possible = km_possible(pr);
    if (path == SLIKL_DK_KEYMAJOR && !possible) return SLIKL_ERR_PARAM_INVALID;
    bool use = false;
    if (possible) {
        const int64_t s2m = (key_range_bound(pr) + 255) / 256 * 256;
        // record bytes: the mask words of the heads, then dI (fp32, or a 64-bit fixed-point
        // number in deterministic mode)
        const int rb = pr->N1 > 64 ? 32 : (pr->N1 > 32 || pr->deterministic ? 16 : 8);
        const double rec_bytes = (double)dv->T1 * (double)s2m * rb;
        use = path == SLIKL_DK_KEYMAJOR ||
              (path == SLIKL_DK_AUTO && key_range_bound(pr) <= 16 * pr->topk &&
               rec_bytes <= 8.0 * (1ull << 30));
        if (use) {
            KmShape k{};
            k.km = 1;
            k.S2m = (int)s2m;
            k.kbound = key_range_bound(pr);
            k.rec_bytes = rb;
            k.nkpw = (int)((s2m / 256 + 31) / 32);
            k.units_max = (s2m / 256) * ((dv->T1 + 31) / 32 + pr->B);
            k.qw_bytes = dv->T1 * pr->N1 * pr->D * 2;
            dv->km = k;
        }
    }
    return SLIKL_OK;
}

int current_sm_count(bool *ok) {
    int dev = 0, major = 0, sms = 0;
    *ok = cudaGetDevice(&dev) == cudaSuccess &&
          cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
          major == 10;
    return sms;
}

Params make_params(const slikl_problem *pr, const Derived &dv, const slikl_tensors *tn,
                   void *ws) {
    Params P{};
    P.dtype = pr->dtype;
    P.layout_q = pr->layout_q;
    P.layout_k = pr->layout_k;
    P.deterministic = pr->deterministic;
    P.B = pr->B;
    P.S1 = pr->layout_q == SLIKL_BSND ? pr->S1 : 0;
    P.S2 = pr->layout_k == SLIKL_BSND ? pr->S2 : 0;
    P.T1 = dv.T1;
    P.T2 = dv.T2;
    P.N1 = (int)pr->N1;
    P.D = (int)pr->D;
    P.K = (int)pr->topk;
    if (tn) {
        P.q = tn->q; P.k = tn->k; P.w = tn->w; P.p = tn->attn_softmax_l1norm;
        P.idx = tn->sparse_indices; P.cu_q = tn->cu_seqlens_q; P.cu_k = tn->cu_seqlens_k;
        P.dq = tn->dq; P.dk = tn->dk; P.dw = tn->dw; P.y = tn->softmax_out;
    }
    WsLayout L = make_layout(dv.T1, dv.T2, pr->topk, pr->D, pr->deterministic, dv.km, pr->B);
    char *base = static_cast<char *>(ws);
    P.status = reinterpret_cast<uint32_t *>(base + L.status);
    P.meta = reinterpret_cast<int32_t *>(base + L.meta);
    P.tok_kbase = reinterpret_cast<int32_t *>(base + L.tok_kbase);
    P.tok_klen = reinterpret_cast<int32_t *>(base + L.tok_klen);
    P.tok_cost = reinterpret_cast<int32_t *>(base + L.tok_cost);
    P.tok_tiles = reinterpret_cast<uint64_t *>(base + L.tok_tiles);
    P.cost_prefix = reinterpret_cast<int64_t *>(base + L.cost_prefix);
    P.dk_acc = reinterpret_cast<float *>(base + L.dk_acc);
    P.partials = reinterpret_cast<float *>(base + L.partials);
    P.keys0 = reinterpret_cast<int32_t *>(base + L.keys0);
    P.vals0 = reinterpret_cast<int32_t *>(base + L.vals0);
    P.keys1 = reinterpret_cast<int32_t *>(base + L.keys1);
    P.vals1 = reinterpret_cast<int32_t *>(base + L.vals1);
    P.hist = reinterpret_cast<int32_t *>(base + L.hist);
    P.row_ptr = reinterpret_cast<int32_t *>(base + L.row_ptr);
    P.km = dv.km.km;
    if (P.km) {
        P.S2m = dv.km.S2m;
        P.kbound = dv.km.kbound;
        P.nkpw = dv.km.nkpw;
        P.rec_bytes = dv.km.rec_bytes;
        P.units_max = dv.km.units_max;
        P.tok_pairs = reinterpret_cast<uint32_t *>(base + L.tok_pairs);
        P.rec = base + L.rec;
        P.units = reinterpret_cast<int4 *>(base + L.units);
        P.units_c = reinterpret_cast<int4 *>(base + L.units_c);
        P.unit_off = reinterpret_cast<int64_t *>(base + L.unit_off);
        P.unit_prefix = reinterpret_cast<int64_t *>(base + L.unit_prefix);
        P.km_range = reinterpret_cast<int32_t *>(base + L.km_range);
        P.km_scratch = reinterpret_cast<float *>(base + L.km_scratch);
        P.km_qw = base + L.km_qw;
    }
    return P;
}

slikl_status check_tensors(const slikl_problem *pr, const slikl_tensors *tn, bool need_all) {
    if (!tn) return SLIKL_ERR_PARAM_NULLPTR;
    // a tensor with no elements (TND with T1 = 0 rows of q, or T2 = 0 rows of k) may be NULL:
    // nothing reads or writes it
    const bool q_rows = !(pr->layout_q == SLIKL_TND && pr->T1 == 0);
    const bool k_rows = !(pr->layout_k == SLIKL_TND && pr->T2 == 0);
    if (q_rows && !tn->sparse_indices) return SLIKL_ERR_PARAM_NULLPTR;
    if (pr->layout_q == SLIKL_TND && !tn->cu_seqlens_q) return SLIKL_ERR_PARAM_NULLPTR;
    if (pr->layout_k == SLIKL_TND && !tn->cu_seqlens_k) return SLIKL_ERR_PARAM_NULLPTR;
    if (need_all && q_rows && (!tn->q || !tn->w || !tn->attn_softmax_l1norm || !tn->dq ||
                               !tn->dw || !tn->softmax_out))
        return SLIKL_ERR_PARAM_NULLPTR;
    if (need_all && k_rows && (!tn->k || !tn->dk)) return SLIKL_ERR_PARAM_NULLPTR;
    // 16-byte vector loads/stores of q, k, dq, dk rows; 4-byte elements elsewhere
    auto mis = [](const void *p, uintptr_t a) { return p && (reinterpret_cast<uintptr_t>(p) & (a - 1)); };
    if (mis(tn->q, 16) || mis(tn->k, 16) || mis(tn->dq, 16) || mis(tn->dk, 16) ||
        mis(tn->w, 4) || mis(tn->attn_softmax_l1norm, 4) || mis(tn->sparse_indices, 4) ||
        mis(tn->cu_seqlens_q, 4) || mis(tn->cu_seqlens_k, 4) || mis(tn->dw, 4) ||
        mis(tn->softmax_out, 4))
        return SLIKL_ERR_PARAM_INVALID;
    return SLIKL_OK;
}

// The sparse problem a dense one runs as (reading in include/slikl.h): topk = the row length,
// and for TND keys the row length is the key-range bound the key-major path may assume.
slikl_status dense_to_sparse(const slikl_dense_problem *d, slikl_problem *sp, int64_t *ld_out) {
    if (!d) return SLIKL_ERR_PARAM_NULLPTR;
    if ((d->mask_mode != 0 && d->mask_mode != 3) || d->reserved != 0) return SLIKL_ERR_PARAM_INVALID;
    int64_t ld = d->row_len;
    if (ld == 0 && d->layout_k == SLIKL_BSND) ld = d->S2;
    if (ld < 1 || ld > 8192) return SLIKL_ERR_PARAM_INVALID;
    if (d->layout_k == SLIKL_BSND && ld < d->S2) return SLIKL_ERR_PARAM_INVALID;
    memset(sp, 0, sizeof(*sp));
    sp->dtype = d->dtype;
    sp->layout_q = d->layout_q;
    sp->layout_k = d->layout_k;
    sp->deterministic = d->deterministic;
    sp->B = d->B;
    sp->S1 = d->S1;
    sp->S2 = d->layout_k == SLIKL_BSND ? d->S2 : ld;
    sp->T1 = d->T1;
    sp->T2 = d->T2;
    sp->N1 = d->N1;
    sp->D = d->D;
    sp->topk = ld;
    *ld_out = ld;
    return SLIKL_OK;
}

// Dense workspace: the sparse call's workspace first (its status word at offset 0), then the
// index rows [T1][Ld] int32, then one word for the dense kernel's flag.
struct DenseLayout {
    size_t sparse, idx, flag, total;
};

// The variant that forms p from the main attention: its inputs, checked on the host.
struct MainP {
    const void *q_main, *k_main;
    float *p_out;
    float scale;
    int Nm, Dm;
};

slikl_status check_main(const slikl_main_attention *m) {
    if (!m) return SLIKL_ERR_PARAM_NULLPTR;
    if (m->Nm < 1 || m->Nm > 128 || (m->Dm != 64 && m->Dm != 128) || m->reserved != 0 ||
        !(m->scale == m->scale) || m->scale > 3.0e38f || m->scale < -3.0e38f)
        return SLIKL_ERR_PARAM_INVALID;
    return SLIKL_OK;
}

// Validation, workspace layout and the launch sequence of one call; with mp, the main
// attention's target distribution is formed right after the work split and used as p.
slikl_status run_grad(const slikl_problem *problem, const slikl_tensors *tensors,
                      void *workspace, size_t workspace_bytes, void *stream,
                      const slikl_options *options, const MainP *mp);

}  // namespace

slikl_status dense_layout(const slikl_problem *sp, const slikl_options *options, int64_t ld,
                          DenseLayout *L) {
    size_t sparse = 0;
    slikl_status st = slikl_grad_workspace_size_ex(sp, options, &sparse);
    if (st != SLIKL_OK) return st;
    const int64_t T1 = sp->layout_q == SLIKL_BSND ? sp->B * sp->S1 : sp->T1;
    L->sparse = sparse;
    L->idx = align256(sparse);
    L->flag = align256(L->idx + sizeof(int32_t) * (size_t)T1 * (size_t)ld);
    L->total = L->flag + 256;
    return SLIKL_OK;
}
}  // namespace slikl

using namespace slikl;

extern "C" {

slikl_status slikl_grad_workspace_size_ex(const slikl_problem *problem,
                                          const slikl_options *options, size_t *workspace_bytes) {
    if (!workspace_bytes) return SLIKL_ERR_INNER_NULLPTR;
    Derived dv;
    slikl_status st = validate(problem, &dv);
    if (st != SLIKL_OK) return st;
    st = choose_dk_path(problem, &dv, options ? options->dk_path : SLIKL_DK_AUTO);
    if (st != SLIKL_OK) return st;
    *workspace_bytes = make_layout(dv.T1, dv.T2, problem->topk, problem->D,
                                   problem->deterministic, dv.km, problem->B).total;
    return SLIKL_OK;
}

slikl_status slikl_grad_dk_path(const slikl_problem *problem, const slikl_options *options,
                                int32_t *path) {
    if (!path) return SLIKL_ERR_INNER_NULLPTR;
    Derived dv;
    slikl_status st = validate(problem, &dv);
    if (st != SLIKL_OK) return st;
    st = choose_dk_path(problem, &dv, options ? options->dk_path : SLIKL_DK_AUTO);
    if (st != SLIKL_OK) return st;
    *path = dv.km.km ? SLIKL_DK_KEYMAJOR : SLIKL_DK_SCATTER;
    return SLIKL_OK;
}

slikl_status slikl_grad_workspace_size(const slikl_problem *problem, size_t *workspace_bytes) {
    return slikl_grad_workspace_size_ex(problem, nullptr, workspace_bytes);
}

slikl_status slikl_grad(const slikl_problem *problem, const slikl_tensors *tensors,
                        void *workspace, size_t workspace_bytes, void *stream) {
    return slikl_grad_ex(problem, tensors, workspace, workspace_bytes, stream, nullptr);
}

slikl_status slikl_grad_with_events(const slikl_problem *problem, const slikl_tensors *tensors,
                                    void *workspace, size_t workspace_bytes, void *stream,
                                    void *fused_begin, void *fused_end) {
    slikl_options o{};
    o.dk_path = SLIKL_DK_AUTO;
    o.fused_begin = fused_begin;
    o.fused_end = fused_end;
    return slikl_grad_ex(problem, tensors, workspace, workspace_bytes, stream, &o);
}

slikl_status slikl_grad_ex(const slikl_problem *problem, const slikl_tensors *tensors,
                           void *workspace, size_t workspace_bytes, void *stream,
                           const slikl_options *options) {
    return run_grad(problem, tensors, workspace, workspace_bytes, stream, options, nullptr);
}

slikl_status slikl_grad_recompute_p_workspace_size(const slikl_problem *problem,
                                                   const slikl_main_attention *main,
                                                   const slikl_options *options,
                                                   size_t *workspace_bytes) {
    const slikl_status st = check_main(main);
    if (st != SLIKL_OK) return st;
    return slikl_grad_workspace_size_ex(problem, options, workspace_bytes);
}

slikl_status slikl_grad_recompute_p(const slikl_problem *problem, const slikl_main_attention *main,
                                    const slikl_tensors *tensors, const void *q_main,
                                    const void *k_main, float *p_out, void *workspace,
                                    size_t workspace_bytes, void *stream,
                                    const slikl_options *options) {
    slikl_status st = check_main(main);
    if (st != SLIKL_OK) return st;
    Derived dv;
    st = validate(problem, &dv);
    if (st != SLIKL_OK) return st;
    if (!tensors) return SLIKL_ERR_PARAM_NULLPTR;
    if ((dv.T1 > 0 && (!q_main || !p_out)) || (dv.T2 > 0 && !k_main)) return SLIKL_ERR_PARAM_NULLPTR;
    if ((reinterpret_cast<uintptr_t>(q_main) & 15) || (reinterpret_cast<uintptr_t>(k_main) & 15) ||
        (reinterpret_cast<uintptr_t>(p_out) & 3))
        return SLIKL_ERR_PARAM_INVALID;
    slikl_tensors tn = *tensors;
    tn.attn_softmax_l1norm = p_out;            // the computed p is the backward's target
    const MainP mp{q_main, k_main, p_out, main->scale, main->Nm, main->Dm};
    return run_grad(problem, &tn, workspace, workspace_bytes, stream, options, &mp);
}

}  // extern "C"

namespace slikl {
namespace {

slikl_status run_grad(const slikl_problem *problem, const slikl_tensors *tensors,
                      void *workspace, size_t workspace_bytes, void *stream,
                      const slikl_options *options, const MainP *mp) {
    Derived dv;
    slikl_status st = validate(problem, &dv);
    if (st != SLIKL_OK) return st;
    st = choose_dk_path(problem, &dv, options ? options->dk_path : SLIKL_DK_AUTO);
    if (st != SLIKL_OK) return st;
    st = check_tensors(problem, tensors, true);
    if (st != SLIKL_OK) return st;
    if (options && ((reinterpret_cast<uintptr_t>(options->loss) & 3) ||
                    (reinterpret_cast<uintptr_t>(options->seq_used_q) & 3) ||
                    (reinterpret_cast<uintptr_t>(options->seq_used_k) & 3)))
        return SLIKL_ERR_PARAM_INVALID;
    if (!workspace) return SLIKL_ERR_PARAM_NULLPTR;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return SLIKL_ERR_PARAM_INVALID;
    WsLayout L = make_layout(dv.T1, dv.T2, problem->topk, problem->D, problem->deterministic,
                             dv.km, problem->B);
    if (workspace_bytes < L.total) return SLIKL_ERR_WORKSPACE_TOO_SMALL;
    bool ok = false;
    int sms = current_sm_count(&ok);
    if (!ok) return SLIKL_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Params P = make_params(problem, dv, tensors, workspace);
    if (options) {
        P.used_q = options->seq_used_q;
        P.used_k = options->seq_used_k;
    }
    void *fused_begin = options ? options->fused_begin : nullptr;
    void *fused_end = options ? options->fused_end : nullptr;

    const int workers = sms < kMaxWorkers ? sms : kMaxWorkers;
    if (cudaMemsetAsync(P.status, 0, 256, s) != cudaSuccess) return SLIKL_ERR_CUDA;
    // deterministic mode on the scatter path: sorted per-slot rows; otherwise the fp32 rows
    const bool sorted = P.deterministic && !P.km;
    // the key-major kernel's CTAs (its deterministic scratch holds kKmDetWorkers of them)
    const int km_workers = P.deterministic && workers > kKmDetWorkers ? kKmDetWorkers : workers;
    if (!sorted && dv.T2 > 0 &&
        cudaMemsetAsync(P.dk_acc, 0, sizeof(float) * (size_t)dv.T2 * problem->D, s) != cudaSuccess)
        return SLIKL_ERR_CUDA;
    if (launch_metadata(P, workers, 1, s) != cudaSuccess) return SLIKL_ERR_CUDA;
    if (P.km && launch_km_metadata(P, km_workers, s) != cudaSuccess) return SLIKL_ERR_CUDA;
    if (mp && launch_main_p(P, mp->q_main, mp->k_main, mp->p_out, mp->scale, mp->Nm, mp->Dm,
                            workers, s) != cudaSuccess)
        return SLIKL_ERR_CUDA;
    if (fused_begin && cudaEventRecord(static_cast<cudaEvent_t>(fused_begin), s) != cudaSuccess)
        return SLIKL_ERR_CUDA;
    if (dv.T1 > 0 && launch_fused_sm100(P, workers, s) != cudaSuccess) return SLIKL_ERR_CUDA;
    if (fused_end && cudaEventRecord(static_cast<cudaEvent_t>(fused_end), s) != cudaSuccess)
        return SLIKL_ERR_CUDA;
    if (options && options->loss && launch_kl_loss(P, options->loss, s) != cudaSuccess)
        return SLIKL_ERR_CUDA;
    void *dk_begin = options ? options->dk_begin : nullptr;
    void *dk_end = options ? options->dk_end : nullptr;
    if (dk_begin && cudaEventRecord(static_cast<cudaEvent_t>(dk_begin), s) != cudaSuccess)
        return SLIKL_ERR_CUDA;
    if (P.km && dv.T1 > 0) {
        if (launch_dk_keymajor(P, km_workers, s) != cudaSuccess) return SLIKL_ERR_CUDA;
        if (P.deterministic && launch_km_det_combine(P, km_workers, s) != cudaSuccess)
            return SLIKL_ERR_CUDA;
    }
    cudaError_t e = sorted ? launch_deterministic_reduce(P, s) : launch_cast(P, s);
    if (e != cudaSuccess) return SLIKL_ERR_CUDA;
    if (dk_end && cudaEventRecord(static_cast<cudaEvent_t>(dk_end), s) != cudaSuccess)
        return SLIKL_ERR_CUDA;
    return SLIKL_OK;
}

}  // namespace
}  // namespace slikl

extern "C" {

slikl_status slikl_read_device_status(const void *workspace, void *stream, uint32_t *flags) {
    if (!flags) return SLIKL_ERR_INNER_NULLPTR;
    if (!workspace) return SLIKL_ERR_PARAM_NULLPTR;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SLIKL_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SLIKL_ERR_CUDA;
    *flags = v;
    return SLIKL_OK;
}

int64_t slikl_grad_metadata_size(int32_t num_workers) {
    if (num_workers < 1 || num_workers > kMaxWorkers) return -1;
    return kMetaHeader + 2 * (int64_t)num_workers;
}

slikl_status slikl_grad_metadata_workspace_size(const slikl_problem *problem,
                                                size_t *workspace_bytes) {
    if (!workspace_bytes) return SLIKL_ERR_INNER_NULLPTR;
    Derived dv;
    slikl_status st = validate(problem, &dv);
    if (st != SLIKL_OK) return st;
    // the metadata kernels touch the regions up to and including cost_prefix
    *workspace_bytes = make_layout(dv.T1, dv.T2, problem->topk, problem->D, 1).dk_acc;
    return SLIKL_OK;
}

slikl_status slikl_grad_metadata(const slikl_problem *problem, const slikl_tensors *tensors,
                                 int32_t num_workers, int32_t mode, int32_t *metadata,
                                 void *workspace, size_t workspace_bytes, void *stream) {
    Derived dv;
    slikl_status st = validate(problem, &dv);
    if (st != SLIKL_OK) return st;
    st = check_tensors(problem, tensors, false);
    if (st != SLIKL_OK) return st;
    if (!metadata || !workspace) return SLIKL_ERR_PARAM_NULLPTR;
    if (num_workers < 1 || num_workers > kMaxWorkers || (mode != 0 && mode != 1))
        return SLIKL_ERR_PARAM_INVALID;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return SLIKL_ERR_PARAM_INVALID;
    size_t need = make_layout(dv.T1, dv.T2, problem->topk, problem->D, 1).dk_acc;
    if (workspace_bytes < need) return SLIKL_ERR_WORKSPACE_TOO_SMALL;
    bool ok = false;
    current_sm_count(&ok);
    if (!ok) return SLIKL_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Params P = make_params(problem, dv, tensors, workspace);
    if (cudaMemsetAsync(P.status, 0, 256, s) != cudaSuccess) return SLIKL_ERR_CUDA;
    if (launch_metadata(P, num_workers, mode, s) != cudaSuccess) return SLIKL_ERR_CUDA;
    size_t bytes = sizeof(int32_t) * (size_t)(kMetaHeader + 2 * num_workers);
    if (cudaMemcpyAsync(metadata, P.meta, bytes, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return SLIKL_ERR_CUDA;
    return SLIKL_OK;
}

const char *slikl_status_string(slikl_status status) {
    switch (status) {
        case SLIKL_OK: return "SLIKL_OK";
        case SLIKL_ERR_PARAM_NULLPTR: return "SLIKL_ERR_PARAM_NULLPTR: a required pointer is NULL";
        case SLIKL_ERR_PARAM_INVALID: return "SLIKL_ERR_PARAM_INVALID: parameter outside the supported set";
        case SLIKL_ERR_WORKSPACE_TOO_SMALL: return "SLIKL_ERR_WORKSPACE_TOO_SMALL: workspace below the phase-1 size";
        case SLIKL_ERR_INNER_NULLPTR: return "SLIKL_ERR_INNER_NULLPTR: output pointer is NULL";
        case SLIKL_ERR_CUDA: return "SLIKL_ERR_CUDA: CUDA runtime error or no sm_100 device";
        default: return "unknown slikl status";
    }
}


slikl_status slikl_dense_grad_workspace_size(const slikl_dense_problem *problem,
                                             const slikl_options *options,
                                             size_t *workspace_bytes) {
    if (!workspace_bytes) return SLIKL_ERR_INNER_NULLPTR;
    slikl_problem sp;
    int64_t ld = 0;
    slikl_status st = dense_to_sparse(problem, &sp, &ld);
    if (st != SLIKL_OK) return st;
    DenseLayout L;
    st = dense_layout(&sp, options, ld, &L);
    if (st != SLIKL_OK) return st;
    *workspace_bytes = L.total;
    return SLIKL_OK;
}

slikl_status slikl_dense_grad_dk_path(const slikl_dense_problem *problem,
                                      const slikl_options *options, int32_t *path) {
    slikl_problem sp;
    int64_t ld = 0;
    slikl_status st = dense_to_sparse(problem, &sp, &ld);
    if (st != SLIKL_OK) return st;
    return slikl_grad_dk_path(&sp, options, path);
}

slikl_status slikl_dense_grad(const slikl_dense_problem *problem,
                              const slikl_dense_tensors *tensors, void *workspace,
                              size_t workspace_bytes, void *stream,
                              const slikl_options *options) {
    slikl_problem sp;
    int64_t ld = 0;
    slikl_status st = dense_to_sparse(problem, &sp, &ld);
    if (st != SLIKL_OK) return st;
    DenseLayout L;
    st = dense_layout(&sp, options, ld, &L);
    if (st != SLIKL_OK) return st;
    if (!tensors) return SLIKL_ERR_PARAM_NULLPTR;
    if (!workspace) return SLIKL_ERR_PARAM_NULLPTR;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return SLIKL_ERR_PARAM_INVALID;
    if (workspace_bytes < L.total) return SLIKL_ERR_WORKSPACE_TOO_SMALL;
    char *ws = static_cast<char *>(workspace);
    slikl_tensors tn;
    tn.q = tensors->q;
    tn.k = tensors->k;
    tn.w = tensors->w;
    tn.attn_softmax_l1norm = tensors->attn_softmax_l1norm;
    tn.sparse_indices = reinterpret_cast<const int32_t *>(ws + L.idx);
    tn.cu_seqlens_q = tensors->cu_seqlens_q;
    tn.cu_seqlens_k = tensors->cu_seqlens_k;
    tn.dq = tensors->dq;
    tn.dk = tensors->dk;
    tn.dw = tensors->dw;
    tn.softmax_out = tensors->softmax_out;
    // every host-side check of the sparse call first, so that nothing is launched for a call
    // that the sparse entry point would reject
    Derived dv;
    st = validate(&sp, &dv);
    if (st != SLIKL_OK) return st;
    st = check_tensors(&sp, &tn, true);
    if (st != SLIKL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t *flag = reinterpret_cast<uint32_t *>(ws + L.flag);
    if (cudaMemsetAsync(flag, 0, 4, s) != cudaSuccess) return SLIKL_ERR_CUDA;
    if (launch_dense_indices(reinterpret_cast<int32_t *>(ws + L.idx), dv.T1, sp.B,
                             sp.layout_q == SLIKL_BSND ? sp.S1 : 0,
                             sp.layout_k == SLIKL_BSND ? sp.S2 : 0, (int)ld, sp.layout_q,
                             sp.layout_k, problem->mask_mode, tn.cu_seqlens_q, tn.cu_seqlens_k,
                             options ? options->seq_used_q : nullptr,
                             options ? options->seq_used_k : nullptr, flag, s) != cudaSuccess)
        return SLIKL_ERR_CUDA;
    st = slikl_grad_ex(&sp, &tn, workspace, L.sparse, stream, options);
    if (st != SLIKL_OK) return st;
    if (launch_dense_flag_merge(flag, reinterpret_cast<uint32_t *>(ws), s) != cudaSuccess)
        return SLIKL_ERR_CUDA;
    return SLIKL_OK;
}

}  // extern "C"
