/*
 * abi_check.c -- a plain C99 client of include/indexcache.h.
 *
 * Built and run by tests/test_c_abi_cpu.py on a host without a GPU.  It
 * proves the header is a C header (not only C++), that a C program links
 * against the library, and it prints, as one JSON object, the size and field
 * offsets of every struct of the ABI plus the results of calls that must
 * return before any device access.  The test compares the layouts with the
 * Python binding's ctypes structures.
 */
#include <stddef.h>
#include <stdio.h>
#include <string.h>

#include "indexcache.h"

#define FIELD(T, f) printf("\"%s\": %zu, ", #f, offsetof(T, f))

int main(void) {
    ic_rows rows = {1, 16, 0, 16};
    ic_stack_shape shape;
    ic_layer_io layers[2];
    int32_t idx_host[64];
    unsigned char ws_host[4096 + 256];
    void* ws = (void*)(((size_t)ws_host + 255) / 256 * 256);
    ic_status bad_pattern, short_pattern, no_ws, bad_k, bad_page_size, paged_no_ws;
    ic_paged_rows paged;

    memset(&shape, 0, sizeof(shape));
    shape.rows = rows;
    shape.H_I = 4;
    shape.d_I = 32;
    shape.idx_dtype = IC_F32;
    shape.k = 4;
    shape.Hq = 8;
    shape.d_qk = 64;
    shape.d_v = 64;
    shape.attn_dtype = IC_F32;
    shape.k_row_stride = 64;
    shape.v_row_stride = 64;
    shape.scale = 0.125f;
    memset(layers, 0, sizeof(layers));

    /* host memory stands in for device buffers: every call below must be
     * rejected by argument checks before it reaches the device */
    bad_pattern = ic_layer_stack_forward("SF", 2, layers, &shape, idx_host, NULL, ws, 4096, NULL);
    short_pattern = ic_layer_stack_forward("F", 2, layers, &shape, idx_host, NULL, ws, 4096, NULL);
    no_ws = ic_topk((const float*)ws, 16, rows, 4, idx_host, NULL, 0, NULL);
    bad_k = ic_topk((const float*)ws, 16, rows, 0, idx_host, ws, 4096, NULL);
    /* a page size that is not a multiple of 128, then a missing workspace */
    memset(&paged, 0, sizeof(paged));
    paged.B = 2; paged.Lq = 1; paged.T_max = 512; paged.seq_lens = idx_host;
    paged.block_table = idx_host; paged.max_pages = 4; paged.page_size = 100; paged.num_pages = 8;
    bad_page_size = ic_sparse_attn_paged(ws, ws, idx_host, 4, &paged, 0.1f, ws, ws, 4096, NULL);
    paged.page_size = 128;
    paged_no_ws = ic_sparse_attn_paged(ws, ws, idx_host, 4, &paged, 0.1f, ws, NULL, 0, NULL);

    printf("{");
    printf("\"ic_rows\": {\"size\": %zu, ", sizeof(ic_rows));
    FIELD(ic_rows, B); FIELD(ic_rows, Lq); FIELD(ic_rows, q_start);
    printf("\"T\": %zu}, ", offsetof(ic_rows, T));
    printf("\"ic_stack_shape\": {\"size\": %zu, ", sizeof(ic_stack_shape));
    FIELD(ic_stack_shape, rows); FIELD(ic_stack_shape, H_I); FIELD(ic_stack_shape, d_I);
    FIELD(ic_stack_shape, idx_dtype); FIELD(ic_stack_shape, k); FIELD(ic_stack_shape, Hq);
    FIELD(ic_stack_shape, d_qk); FIELD(ic_stack_shape, d_v); FIELD(ic_stack_shape, attn_dtype);
    FIELD(ic_stack_shape, k_row_stride); FIELD(ic_stack_shape, v_row_stride);
    printf("\"scale\": %zu}, ", offsetof(ic_stack_shape, scale));
    printf("\"ic_layer_io\": {\"size\": %zu, ", sizeof(ic_layer_io));
    FIELD(ic_layer_io, q_idx); FIELD(ic_layer_io, q_scale); FIELD(ic_layer_io, w);
    FIELD(ic_layer_io, k_idx); FIELD(ic_layer_io, k_scale); FIELD(ic_layer_io, q);
    FIELD(ic_layer_io, kmat); FIELD(ic_layer_io, vmat);
    printf("\"out\": %zu}, ", offsetof(ic_layer_io, out));
    printf("\"ic_paged_rows\": {\"size\": %zu, ", sizeof(ic_paged_rows));
    FIELD(ic_paged_rows, B); FIELD(ic_paged_rows, Lq); FIELD(ic_paged_rows, T_max);
    FIELD(ic_paged_rows, seq_lens); FIELD(ic_paged_rows, block_table);
    FIELD(ic_paged_rows, max_pages); FIELD(ic_paged_rows, page_size);
    printf("\"num_pages\": %zu}, ", offsetof(ic_paged_rows, num_pages));
    printf("\"sizeof_enum\": %zu, ", sizeof(ic_status));
    printf("\"IC_STATUS_BYTES\": %d, ", (int)IC_STATUS_BYTES);
    printf("\"IC_NOALLOC_SCRATCH_BYTES\": %u, ", (unsigned)IC_NOALLOC_SCRATCH_BYTES);
    printf("\"version\": %d, ", ic_version());
    printf("\"ok_string\": \"%s\", ", ic_status_string(IC_OK));
    printf("\"last_error_before\": \"%s\", ", ic_last_error());
    printf("\"bad_pattern\": %d, \"short_pattern\": %d, \"no_ws\": %d, \"bad_k\": %d, ",
           (int)bad_pattern, (int)short_pattern, (int)no_ws, (int)bad_k);
    printf("\"bad_page_size\": %d, \"paged_no_ws\": %d, ", (int)bad_page_size, (int)paged_no_ws);
    printf("\"workspace_size\": %zu, ", ic_workspace_size(&shape));
    printf("\"launches\": %llu", (unsigned long long)ic_kernel_launches(0));
    printf("}\n");
    return 0;
}
