/* Plain C11 use of include/pagedattn.h: host-only entry points of
 * libpagedattn (no GPU needed).  tests/test_abi.py compiles it with
 * -std=c11 -pedantic -Werror, links it against the library, runs it and
 * compares its output with the same calls made through the Python binding. */
#include <stddef.h>
#include <stdio.h>
#include <string.h>

#include "pagedattn.h"

int main(void)
{
    /* a decode row, an MTP row and a short prefill chunk, per-row windows */
    const int32_t seq_lens[3] = {300, 40, 7};
    const int32_t query_lens[3] = {5, 1, 3};
    const int32_t windows[3] = {16, 100, 2};
    int span = 0, qlen = 0;
    if (pa_extents_host(seq_lens, query_lens, windows, 0, 3, &span, &qlen) != PA_OK) {
        fprintf(stderr, "extents: %s\n", pa_last_error());
        return 1;
    }
    pa_params p;
    memset(&p, 0, sizeof p);
    p.batch = 3;
    p.num_q_heads = 8;
    p.num_kv_heads = 2;
    p.head_dim = 128;
    p.num_blocks = 64;
    p.max_blocks_per_seq = 19;
    p.max_span_hint = span;
    p.max_query_len_hint = qlen;
    p.windows = windows;
    pa_plan_info info;
    if (pa_plan(&p, 16, 148, 2, &info) != PA_OK) {
        fprintf(stderr, "plan: %s\n", pa_last_error());
        return 2;
    }
    printf("extents %d %d\n", span, qlen);
    printf("plan %d %d %d %d %d %d %d %d %zu\n", info.variant, info.partition_tokens,
           info.max_partitions, info.one_shot, info.max_rows, info.grid_x, info.grid_y,
           info.grid_z, info.workspace_bytes);
    /* an unsupported head_dim is refused on the host, with a message */
    p.head_dim = 96;
    const int rc = pa_plan(&p, 16, 148, 2, &info);
    printf("refused %d %d\n", rc, (int)(strlen(pa_last_error()) > 0));
    printf("version %s\n", pa_version());
    /* the structs' layout, field by field, for the binding's ctypes mirror */
#define FIELD(T, f) printf("offset " #T "." #f " %zu\n", offsetof(T, f))
    FIELD(pa_params, batch); FIELD(pa_params, num_q_heads); FIELD(pa_params, num_kv_heads);
    FIELD(pa_params, head_dim); FIELD(pa_params, num_blocks);
    FIELD(pa_params, max_blocks_per_seq); FIELD(pa_params, max_span_hint);
    FIELD(pa_params, max_query_len_hint); FIELD(pa_params, windows);
    FIELD(pa_params, workspace); FIELD(pa_params, workspace_bytes);
    FIELD(pa_params, force_variant); FIELD(pa_params, force_partitions);
    FIELD(pa_params, profile_events); FIELD(pa_params, q_dtype); FIELD(pa_params, kv_dtype);
    FIELD(pa_params, q_scale); FIELD(pa_params, k_scale); FIELD(pa_params, v_scale);
    FIELD(pa_params, schedule); FIELD(pa_params, wait_limit_cycles);
    FIELD(pa_params, merge_target_extra);
    FIELD(pa_plan_info, variant); FIELD(pa_plan_info, partition_tokens);
    FIELD(pa_plan_info, max_partitions); FIELD(pa_plan_info, one_shot);
    FIELD(pa_plan_info, max_rows); FIELD(pa_plan_info, slab_rows);
    FIELD(pa_plan_info, consumer_warps); FIELD(pa_plan_info, stages);
    FIELD(pa_plan_info, grid_x); FIELD(pa_plan_info, grid_y); FIELD(pa_plan_info, grid_z);
    FIELD(pa_plan_info, block_threads); FIELD(pa_plan_info, smem_bytes);
    FIELD(pa_plan_info, workspace_bytes); FIELD(pa_plan_info, num_sms);
    FIELD(pa_plan_info, ctas_per_sm); FIELD(pa_plan_info, worklist);
#undef FIELD
    printf("sizeof pa_params %zu\n", sizeof(pa_params));
    printf("sizeof pa_plan_info %zu\n", sizeof(pa_plan_info));
    return 0;
}
