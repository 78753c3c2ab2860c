/*
 * A plain C11 client of include/ep_b200.h: no torch, only the CUDA runtime
 * for device memory.  Test infrastructure for tests/test_gpu_c_abi.py, which
 * writes the inputs, runs this program and compares its outputs with the
 * oracle.
 *
 *   c_abi_client <dir> T K E R A H
 *
 * Reads <dir>/topk_idx.bin (int64 [T, K]), <dir>/topk_weights.bin (fp32
 * [T, K]), <dir>/x.bin (bf16 bits [T, H]) and <dir>/y.bin (bf16 bits
 * [capacity, H], the expert outputs).  Runs ep_layout, ep_dispatch (zero
 * padding) and ep_combine (weighted) on a caller-allocated workspace, then
 * ep_layout_no_alloc on the same inputs, then one source group into R
 * separately allocated regions (ep_layout with alignment 1,
 * ep_source_offsets, ep_dispatch_regions with the padding list,
 * ep_combine_regions), and writes pair_slot.bin, expert_offset.bin, recv.bin
 * (the first expert_offset[E] rows), out.bin, pair_slot_no_alloc.bin,
 * regions.bin (the regions' rows one after the other) and out_regions.bin.  Exit status 0 on success; any library or CUDA
 * error prints its status string and exits 1.
 */
#include <cuda_runtime_api.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "ep_b200.h"

static void* read_file(const char* dir, const char* name, size_t bytes)
{
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE* f = fopen(path, "rb");
    if (!f) {
        fprintf(stderr, "cannot open %s\n", path);
        exit(1);
    }
    void* p = malloc(bytes ? bytes : 1);
    if (!p || fread(p, 1, bytes, f) != bytes) {
        fprintf(stderr, "short read of %s\n", path);
        exit(1);
    }
    fclose(f);
    return p;
}

static void write_file(const char* dir, const char* name, const void* p, size_t bytes)
{
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE* f = fopen(path, "wb");
    if (!f || fwrite(p, 1, bytes, f) != bytes) {
        fprintf(stderr, "cannot write %s\n", path);
        exit(1);
    }
    fclose(f);
}

static void check_cuda(cudaError_t e, const char* what)
{
    if (e != cudaSuccess) {
        fprintf(stderr, "%s: %s\n", what, cudaGetErrorString(e));
        exit(1);
    }
}

static void check_ep(int rc, const char* what)
{
    if (rc != EP_OK) {
        fprintf(stderr, "%s: %s (%d)\n", what, ep_status_string(rc), rc);
        exit(1);
    }
}

static void* dev_alloc(size_t bytes)
{
    void* p = NULL;
    check_cuda(cudaMalloc(&p, bytes ? bytes : 16), "cudaMalloc");
    return p;
}

static void* dev_copy(const void* host, size_t bytes)
{
    void* p = dev_alloc(bytes);
    check_cuda(cudaMemcpy(p, host, bytes, cudaMemcpyHostToDevice), "H2D");
    return p;
}

int main(int argc, char** argv)
{
    if (argc != 8) {
        fprintf(stderr, "usage: %s dir T K E R A H\n", argv[0]);
        return 2;
    }
    const char* dir = argv[1];
    const int T = atoi(argv[2]), K = atoi(argv[3]), E = atoi(argv[4]), R = atoi(argv[5]), A = atoi(argv[6]),
              H = atoi(argv[7]);
    if (ep_version() != EP_B200_VERSION) {
        fprintf(stderr, "header version %d, library version %d\n", EP_B200_VERSION, ep_version());
        return 1;
    }
    const int64_t cap = ep_capacity_rows(T, K, E, A);
    const size_t ws_bytes = ep_workspace_bytes(T, K, E, A);
    if (cap <= 0 || ws_bytes == 0) {
        fprintf(stderr, "bad sizes\n");
        return 1;
    }

    int64_t* h_idx = (int64_t*)read_file(dir, "topk_idx.bin", (size_t)T * K * 8);
    float* h_w = (float*)read_file(dir, "topk_weights.bin", (size_t)T * K * 4);
    uint16_t* h_x = (uint16_t*)read_file(dir, "x.bin", (size_t)T * H * 2);
    uint16_t* h_y = (uint16_t*)read_file(dir, "y.bin", (size_t)cap * H * 2);

    int64_t* d_idx = (int64_t*)dev_copy(h_idx, (size_t)T * K * 8);
    float* d_w = (float*)dev_copy(h_w, (size_t)T * K * 4);
    void* d_x = dev_copy(h_x, (size_t)T * H * 2);
    void* d_y = dev_copy(h_y, (size_t)cap * H * 2);
    void* d_recv = dev_alloc((size_t)cap * H * 2);
    void* d_out = dev_alloc((size_t)T * H * 2);

    ep_layout_t lay;
    memset(&lay, 0, sizeof lay);
    lay.num_recv_tokens_per_expert = (int32_t*)dev_alloc((size_t)E * 4);
    lay.expert_offset = (int32_t*)dev_alloc((size_t)(E + 1) * 4);
    lay.pair_slot = (int32_t*)dev_alloc((size_t)T * K * 4);
    lay.recv_src_token = (int32_t*)dev_alloc((size_t)cap * 4);
    lay.recv_weight = (float*)dev_alloc((size_t)cap * 4);
    lay.recv_local_expert = (int32_t*)dev_alloc((size_t)cap * 4);
    lay.workspace = dev_alloc(ws_bytes);
    lay.workspace_bytes = ws_bytes;
    lay.capacity = cap;
    check_cuda(cudaMemset(lay.workspace, 0, ws_bytes), "workspace zero-fill");

    check_ep(ep_layout(d_idx, d_w, T, K, E, R, A, 0, &lay, NULL), "ep_layout");
    check_ep(ep_dispatch(&lay, d_x, EP_DTYPE_BF16, NULL, H, 0, 0, 1, d_recv, NULL, NULL), "ep_dispatch");
    check_ep(ep_combine(&lay, d_y, H, d_w, NULL, NULL, d_out, NULL), "ep_combine");
    uint32_t flags = 0;
    check_ep(ep_get_status(&lay, NULL, &flags), "ep_get_status");

    int32_t* h_slot = (int32_t*)malloc((size_t)T * K * 4 + 4);
    int32_t* h_off = (int32_t*)malloc((size_t)(E + 1) * 4);
    check_cuda(cudaMemcpy(h_slot, lay.pair_slot, (size_t)T * K * 4, cudaMemcpyDeviceToHost), "D2H slots");
    check_cuda(cudaMemcpy(h_off, lay.expert_offset, (size_t)(E + 1) * 4, cudaMemcpyDeviceToHost), "D2H off");
    const int64_t rows = h_off[E];
    uint16_t* h_recv = (uint16_t*)malloc((size_t)(rows > 0 ? rows : 1) * H * 2);
    uint16_t* h_out = (uint16_t*)malloc((size_t)T * H * 2 + 2);
    check_cuda(cudaMemcpy(h_recv, d_recv, (size_t)rows * H * 2, cudaMemcpyDeviceToHost), "D2H recv");
    check_cuda(cudaMemcpy(h_out, d_out, (size_t)T * H * 2, cudaMemcpyDeviceToHost), "D2H out");
    write_file(dir, "pair_slot.bin", h_slot, (size_t)T * K * 4);
    write_file(dir, "expert_offset.bin", h_off, (size_t)(E + 1) * 4);
    write_file(dir, "recv.bin", h_recv, (size_t)rows * H * 2);
    write_file(dir, "out.bin", h_out, (size_t)T * H * 2);

    /* the same layout with the library-owned workspace */
    ep_layout_t lay2 = lay;
    lay2.workspace = NULL;
    lay2.workspace_bytes = 0;
    check_cuda(cudaMemset(lay2.pair_slot, 0xff, (size_t)T * K * 4), "clear slots");
    check_ep(ep_layout_no_alloc(d_idx, d_w, T, K, E, R, A, 0, &lay2, NULL), "ep_layout_no_alloc");
    check_ep(ep_get_status(&lay2, NULL, &flags), "ep_get_status (no-alloc)");
    check_cuda(cudaMemcpy(h_slot, lay2.pair_slot, (size_t)T * K * 4, cudaMemcpyDeviceToHost), "D2H slots 2");
    write_file(dir, "pair_slot_no_alloc.bin", h_slot, (size_t)T * K * 4);

    /* one source group into R separately allocated regions: an alignment-1
       layout of the same tokens, the offsets from its counts, then dispatch
       and combine over a device table of region addresses */
    ep_layout_t lay3 = lay;
    const int64_t cap1 = ep_capacity_rows(T, K, E, 1);
    lay3.pair_slot = (int32_t*)dev_alloc((size_t)T * K * 4);
    lay3.num_recv_tokens_per_expert = (int32_t*)dev_alloc((size_t)E * 4);
    lay3.expert_offset = (int32_t*)dev_alloc((size_t)(E + 1) * 4);
    lay3.recv_src_token = (int32_t*)dev_alloc((size_t)cap1 * 4);
    lay3.recv_weight = (float*)dev_alloc((size_t)cap1 * 4);
    lay3.recv_local_expert = (int32_t*)dev_alloc((size_t)cap1 * 4);
    lay3.capacity = cap1;
    lay3.workspace_bytes = ep_workspace_bytes(T, K, E, 1);
    lay3.workspace = dev_alloc(lay3.workspace_bytes);
    check_cuda(cudaMemset(lay3.workspace, 0, lay3.workspace_bytes), "workspace 3 zero-fill");
    check_ep(ep_layout(d_idx, d_w, T, K, E, R, 1, 0, &lay3, NULL), "ep_layout (alignment 1)");
    int32_t* h_cnt = (int32_t*)malloc((size_t)E * 4);
    check_cuda(cudaMemcpy(h_cnt, lay3.num_recv_tokens_per_expert, (size_t)E * 4, cudaMemcpyDeviceToHost), "D2H cnt");
    int32_t* h_delta = (int32_t*)malloc((size_t)E * 4);
    int64_t* h_rows = (int64_t*)malloc((size_t)R * 8);
    int64_t npad = 0;
    check_ep(ep_source_offsets(h_cnt, 1, E, R, A, 0, h_delta, h_rows, NULL, 0, &npad), "ep_source_offsets");
    int64_t* h_pads = (int64_t*)malloc((size_t)(npad > 0 ? npad : 1) * 8);
    check_ep(ep_source_offsets(h_cnt, 1, E, R, A, 0, h_delta, h_rows, h_pads, npad, &npad), "ep_source_offsets");
    int64_t rcap = 1;
    for (int r = 0; r < R; ++r) rcap = h_rows[r] > rcap ? h_rows[r] : rcap;
    void** h_reg = (void**)malloc((size_t)R * sizeof(void*));
    void** h_yreg = (void**)malloc((size_t)R * sizeof(void*));
    int64_t base = 0;
    for (int r = 0; r < R; ++r) {
        h_reg[r] = dev_alloc((size_t)rcap * H * 2);
        h_yreg[r] = dev_alloc((size_t)rcap * H * 2);
        /* the expert outputs of region r: its rows of the single receive order */
        check_cuda(cudaMemcpy(h_yreg[r], h_y + (size_t)base * H, (size_t)h_rows[r] * H * 2, cudaMemcpyHostToDevice),
                   "H2D y region");
        base += h_rows[r];
    }
    void* d_reg = dev_copy(h_reg, (size_t)R * sizeof(void*));
    void* d_yreg = dev_copy(h_yreg, (size_t)R * sizeof(void*));
    void* d_delta = dev_copy(h_delta, (size_t)E * 4);
    void* d_pads = dev_copy(h_pads, (size_t)(npad > 0 ? npad : 1) * 8);
    void* d_out2 = dev_alloc((size_t)T * H * 2);
    check_ep(ep_dispatch_regions(&lay3, d_idx, (const int32_t*)d_delta, (void* const*)d_reg, rcap, d_x, H,
                                 (const int64_t*)d_pads, npad, NULL), "ep_dispatch_regions");
    check_ep(ep_combine_regions(&lay3, d_idx, (const int32_t*)d_delta, (const void* const*)d_yreg, rcap, H, d_w,
                                d_out2, NULL), "ep_combine_regions");
    check_ep(ep_get_status(&lay3, NULL, &flags), "ep_get_status (regions)");
    uint16_t* h_regs = (uint16_t*)malloc((size_t)(base > 0 ? base : 1) * H * 2);
    int64_t at = 0;
    for (int r = 0; r < R; ++r) {
        check_cuda(cudaMemcpy(h_regs + (size_t)at * H, h_reg[r], (size_t)h_rows[r] * H * 2, cudaMemcpyDeviceToHost),
                   "D2H region");
        at += h_rows[r];
    }
    write_file(dir, "regions.bin", h_regs, (size_t)base * H * 2);
    check_cuda(cudaMemcpy(h_out, d_out2, (size_t)T * H * 2, cudaMemcpyDeviceToHost), "D2H out 2");
    write_file(dir, "out_regions.bin", h_out, (size_t)T * H * 2);

    printf("ok rows=%lld\n", (long long)rows);
    return 0;
}
