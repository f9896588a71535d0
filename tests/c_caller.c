/*
 * A plain C99 caller of the library's C ABI (include/slikl.h), built and run by
 * tests/test_c_caller.py on the host (no GPU needed: phase 1 and the host-side checks make no
 * CUDA call).
 *
 * It prints the size and field offsets of every struct of the ABI, as this C compiler lays
 * them out, and the phase-1 results for the problems given on the command line, one per
 * argument as "dtype,layout,B,S1,S2,T1,T2,N1,D,topk,deterministic,dk_path".
 */
#include <stddef.h>
#include <stdio.h>
#include <stdlib.h>

#include "slikl.h"

#define FIELD(T, f) printf("field " #T " " #f " %zu\n", offsetof(T, f))

static void layouts(void) {
    printf("size slikl_problem %zu\n", sizeof(slikl_problem));
    FIELD(slikl_problem, dtype); FIELD(slikl_problem, layout_q); FIELD(slikl_problem, layout_k);
    FIELD(slikl_problem, deterministic); FIELD(slikl_problem, B); FIELD(slikl_problem, S1);
    FIELD(slikl_problem, S2); FIELD(slikl_problem, T1); FIELD(slikl_problem, T2);
    FIELD(slikl_problem, N1); FIELD(slikl_problem, D); FIELD(slikl_problem, topk);
    printf("size slikl_tensors %zu\n", sizeof(slikl_tensors));
    FIELD(slikl_tensors, q); FIELD(slikl_tensors, k); FIELD(slikl_tensors, w);
    FIELD(slikl_tensors, attn_softmax_l1norm); FIELD(slikl_tensors, sparse_indices);
    FIELD(slikl_tensors, cu_seqlens_q); FIELD(slikl_tensors, cu_seqlens_k);
    FIELD(slikl_tensors, dq); FIELD(slikl_tensors, dk); FIELD(slikl_tensors, dw);
    FIELD(slikl_tensors, softmax_out);
    printf("size slikl_options %zu\n", sizeof(slikl_options));
    FIELD(slikl_options, dk_path); FIELD(slikl_options, fused_begin);
    FIELD(slikl_options, fused_end); FIELD(slikl_options, dk_begin); FIELD(slikl_options, dk_end);
    FIELD(slikl_options, loss); FIELD(slikl_options, seq_used_q); FIELD(slikl_options, seq_used_k);
    printf("size slikl_dense_problem %zu\n", sizeof(slikl_dense_problem));
    FIELD(slikl_dense_problem, dtype); FIELD(slikl_dense_problem, layout_q);
    FIELD(slikl_dense_problem, layout_k); FIELD(slikl_dense_problem, deterministic);
    FIELD(slikl_dense_problem, B); FIELD(slikl_dense_problem, S1); FIELD(slikl_dense_problem, S2);
    FIELD(slikl_dense_problem, T1); FIELD(slikl_dense_problem, T2); FIELD(slikl_dense_problem, N1);
    FIELD(slikl_dense_problem, D); FIELD(slikl_dense_problem, row_len);
    FIELD(slikl_dense_problem, mask_mode); FIELD(slikl_dense_problem, reserved);
    printf("size slikl_dense_tensors %zu\n", sizeof(slikl_dense_tensors));
    FIELD(slikl_dense_tensors, q); FIELD(slikl_dense_tensors, k); FIELD(slikl_dense_tensors, w);
    FIELD(slikl_dense_tensors, attn_softmax_l1norm); FIELD(slikl_dense_tensors, cu_seqlens_q);
    FIELD(slikl_dense_tensors, cu_seqlens_k); FIELD(slikl_dense_tensors, dq);
    FIELD(slikl_dense_tensors, dk); FIELD(slikl_dense_tensors, dw);
    FIELD(slikl_dense_tensors, softmax_out);
    printf("size slikl_main_attention %zu\n", sizeof(slikl_main_attention));
    FIELD(slikl_main_attention, Nm); FIELD(slikl_main_attention, Dm);
    FIELD(slikl_main_attention, scale); FIELD(slikl_main_attention, reserved);
}

int main(int argc, char **argv) {
    layouts();
    for (int i = 1; i < argc; ++i) {
        slikl_problem p;
        slikl_options o = {0};
        long long v[12];
        if (sscanf(argv[i], "%lld,%lld,%lld,%lld,%lld,%lld,%lld,%lld,%lld,%lld,%lld,%lld",
                   &v[0], &v[1], &v[2], &v[3], &v[4], &v[5], &v[6], &v[7], &v[8], &v[9],
                   &v[10], &v[11]) != 12) {
            fprintf(stderr, "bad problem argument: %s\n", argv[i]);
            return 2;
        }
        p.dtype = (int32_t)v[0];
        p.layout_q = p.layout_k = (int32_t)v[1];
        p.B = v[2]; p.S1 = v[3]; p.S2 = v[4]; p.T1 = v[5]; p.T2 = v[6];
        p.N1 = v[7]; p.D = v[8]; p.topk = v[9]; p.deterministic = (int32_t)v[10];
        o.dk_path = (int32_t)v[11];
        size_t plain = 0, ex = 0;
        int32_t path = -1;
        slikl_status a = slikl_grad_workspace_size(&p, &plain);
        slikl_status b = slikl_grad_workspace_size_ex(&p, &o, &ex);
        slikl_status c = slikl_grad_dk_path(&p, &o, &path);
        printf("problem %d %d %d %zu %zu %d\n", (int)a, (int)b, (int)c, plain, ex, (int)path);
    }
    printf("status %d %s\n", (int)SLIKL_ERR_PARAM_INVALID,
           slikl_status_string(SLIKL_ERR_PARAM_INVALID));
    return 0;
}
