/* A plain C99 program that drives the device path of the C ABI on its own:
 * it allocates every device buffer itself (the library allocates none),
 * creates a non-default stream, and runs ep_handle_create -> ep_layout ->
 * ep_dispatch (BF16) -> ep_dispatch (FP8 e4m3 1x128) -> ep_combine ->
 * ep_handle_check, then writes the results to a file.  Built and run by
 * tests/test_c_device_consumer.py, which writes the inputs and compares the
 * results with the oracle.
 *
 * Input file (little-endian): int32 T, k, E, R, H, P; int64 topk_idx[T][k];
 * uint16 x[T][H] (bf16 bits); float weights[T][k]; uint16 y[P][H] (the expert
 * outputs in the receive layout, bf16 bits).
 * Output file: int32 status[6] (the status of each call, in the order
 * above), int32 total_recv_rows, int32 expert_off[E+1], int32 dst_row[T][k],
 * int32 recv_src[total], uint16 recv_bf16[total][H], uint8 recv_q[total][H],
 * float recv_scales[total][H/128], uint16 out[T][H].
 * Exit status: 0 when every call returned EP_OK and every CUDA call
 * succeeded; the statuses are in the file either way. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "ep.h"

#define CK(call)                                                                  \
    do {                                                                          \
        cudaError_t e_ = (call);                                                  \
        if (e_ != cudaSuccess) {                                                  \
            fprintf(stderr, "line %d: %s: %s\n", __LINE__, #call, cudaGetErrorString(e_)); \
            return 2;                                                             \
        }                                                                         \
    } while (0)

static int read_all(FILE* f, void* p, size_t n)
{
    return n == 0 || fread(p, 1, n, f) == n;
}

static int write_all(FILE* f, const void* p, size_t n)
{
    return n == 0 || fwrite(p, 1, n, f) == n;
}

int main(int argc, char** argv)
{
    int32_t hdr[6];
    FILE* fin;
    FILE* fout;
    int T, k, E, R, H, P;
    size_t n_idx, n_x, n_y, n_w;
    int64_t* h_idx;
    uint16_t *h_x, *h_y, *h_out, *h_recv;
    float *h_w, *h_scales;
    uint8_t* h_q;
    int32_t *h_off, *h_dst, *h_src;
    void *d_ws, *d_idx, *d_x, *d_y, *d_w, *d_out, *d_recv, *d_q, *d_scales;
    size_t ws_bytes;
    int64_t cap, total_count = 0;
    int32_t total = 0;
    int32_t status[6];
    ep_handle_t h = NULL;
    cudaStream_t s;
    int i, rc = 0;

    if (argc != 3) {
        fprintf(stderr, "usage: %s input output\n", argv[0]);
        return 2;
    }
    fin = fopen(argv[1], "rb");
    if (!fin || !read_all(fin, hdr, sizeof hdr)) {
        fprintf(stderr, "cannot read %s\n", argv[1]);
        return 2;
    }
    T = hdr[0];
    k = hdr[1];
    E = hdr[2];
    R = hdr[3];
    H = hdr[4];
    P = hdr[5];
    n_idx = (size_t)T * k;
    n_x = (size_t)T * H;
    n_y = (size_t)P * H;
    n_w = (size_t)T * k;
    h_idx = (int64_t*)malloc(sizeof(int64_t) * (n_idx ? n_idx : 1));
    h_x = (uint16_t*)malloc(sizeof(uint16_t) * (n_x ? n_x : 1));
    h_w = (float*)malloc(sizeof(float) * (n_w ? n_w : 1));
    h_y = (uint16_t*)malloc(sizeof(uint16_t) * (n_y ? n_y : 1));
    if (!h_idx || !h_x || !h_w || !h_y || !read_all(fin, h_idx, sizeof(int64_t) * n_idx) ||
        !read_all(fin, h_x, sizeof(uint16_t) * n_x) || !read_all(fin, h_w, sizeof(float) * n_w) ||
        !read_all(fin, h_y, sizeof(uint16_t) * n_y)) {
        fprintf(stderr, "short input\n");
        return 2;
    }
    fclose(fin);

    /* device buffers, all owned by this program */
    ws_bytes = ep_workspace_bytes(T, k, E, R, 128);
    cap = ep_recv_rows_upper_bound(T, k, E, 128);
    if (ws_bytes == 0 || cap < P) {
        fprintf(stderr, "bad sizes\n");
        return 2;
    }
    CK(cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking));
    CK(cudaMalloc(&d_ws, ws_bytes));
    CK(cudaMalloc(&d_idx, sizeof(int64_t) * (n_idx ? n_idx : 1)));
    CK(cudaMalloc(&d_x, sizeof(uint16_t) * (n_x ? n_x : 1)));
    CK(cudaMalloc(&d_w, sizeof(float) * (n_w ? n_w : 1)));
    CK(cudaMalloc(&d_y, sizeof(uint16_t) * (size_t)(cap ? cap : 1) * H));
    CK(cudaMalloc(&d_out, sizeof(uint16_t) * (n_x ? n_x : 1)));
    CK(cudaMalloc(&d_recv, sizeof(uint16_t) * (size_t)(cap ? cap : 1) * H));
    CK(cudaMalloc(&d_q, (size_t)(cap ? cap : 1) * H));
    CK(cudaMalloc(&d_scales, sizeof(float) * (size_t)(cap ? cap : 1) * (H / 128)));
    CK(cudaMemcpyAsync(d_idx, h_idx, sizeof(int64_t) * n_idx, cudaMemcpyHostToDevice, s));
    CK(cudaMemcpyAsync(d_x, h_x, sizeof(uint16_t) * n_x, cudaMemcpyHostToDevice, s));
    CK(cudaMemcpyAsync(d_w, h_w, sizeof(float) * n_w, cudaMemcpyHostToDevice, s));
    CK(cudaMemcpyAsync(d_y, h_y, sizeof(uint16_t) * n_y, cudaMemcpyHostToDevice, s));

    /* each call runs only if the ones it needs returned EP_OK; -1 = not run */
    status[0] = (int32_t)ep_handle_create(d_ws, ws_bytes, T, k, E, R, 128, &h);
    status[1] = status[2] = status[3] = status[4] = status[5] = -1;
    if (status[0] == EP_OK) {
        status[1] = (int32_t)ep_layout(h, (const int64_t*)d_idx, T, (void*)s);
        if (status[1] == EP_OK) {
            status[2] = (int32_t)ep_dispatch(h, d_x, H, EP_FMT_BF16, d_recv, NULL, cap, (void*)s);
            status[3] = (int32_t)ep_dispatch(h, d_x, H, EP_FMT_FP8_E4M3_1X128, d_q,
                                             (float*)d_scales, cap, (void*)s);
            status[4] = (int32_t)ep_combine(h, d_y, cap, (const float*)d_w, H, d_out, (void*)s);
        }
        status[5] = (int32_t)ep_handle_check(h, (void*)s);
    }
    for (i = 0; i < 6; ++i)
        if (status[i] != EP_OK) {
            fprintf(stderr, "call %d returned %d (%s): %s\n", i, status[i],
                    ep_strerror((ep_status_t)status[i]), ep_last_error_message());
            rc = 1;
        }

    /* results back to the host */
    h_off = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
    h_dst = (int32_t*)malloc(sizeof(int32_t) * (n_idx ? n_idx : 1));
    h_out = (uint16_t*)malloc(sizeof(uint16_t) * (n_x ? n_x : 1));
    if (!h_off || !h_dst || !h_out)
        return 2;
    memset(h_off, 0, sizeof(int32_t) * (size_t)(E + 1));
    memset(h_dst, 0, sizeof(int32_t) * n_idx);
    memset(h_out, 0, sizeof(uint16_t) * n_x);
    if (status[1] == EP_OK) {
        const void* v_total = ep_handle_view(h, EP_VIEW_TOTAL_RECV_ROWS, &total_count);
        const void* v_off = ep_handle_view(h, EP_VIEW_EXPERT_OFFSET, &total_count);
        const void* v_dst = ep_handle_view(h, EP_VIEW_DST_ROW, &total_count);
        CK(cudaMemcpyAsync(&total, v_total, sizeof total, cudaMemcpyDeviceToHost, s));
        CK(cudaMemcpyAsync(h_off, v_off, sizeof(int32_t) * (size_t)(E + 1),
                           cudaMemcpyDeviceToHost, s));
        CK(cudaMemcpyAsync(h_dst, v_dst, sizeof(int32_t) * n_idx, cudaMemcpyDeviceToHost, s));
        CK(cudaMemcpyAsync(h_out, d_out, sizeof(uint16_t) * n_x, cudaMemcpyDeviceToHost, s));
        CK(cudaStreamSynchronize(s));
    }
    if (total < 0 || total > cap)
        return 2;
    h_src = (int32_t*)malloc(sizeof(int32_t) * (size_t)(total ? total : 1));
    h_recv = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(total ? total : 1) * H);
    h_q = (uint8_t*)malloc((size_t)(total ? total : 1) * H);
    h_scales = (float*)malloc(sizeof(float) * (size_t)(total ? total : 1) * (H / 128));
    if (!h_src || !h_recv || !h_q || !h_scales)
        return 2;
    if (total > 0) {
        const void* v_src = ep_handle_view(h, EP_VIEW_RECV_SRC, &total_count);
        CK(cudaMemcpyAsync(h_src, v_src, sizeof(int32_t) * (size_t)total, cudaMemcpyDeviceToHost, s));
        CK(cudaMemcpyAsync(h_recv, d_recv, sizeof(uint16_t) * (size_t)total * H,
                           cudaMemcpyDeviceToHost, s));
        CK(cudaMemcpyAsync(h_q, d_q, (size_t)total * H, cudaMemcpyDeviceToHost, s));
        CK(cudaMemcpyAsync(h_scales, d_scales, sizeof(float) * (size_t)total * (H / 128),
                           cudaMemcpyDeviceToHost, s));
        CK(cudaStreamSynchronize(s));
    }

    fout = fopen(argv[2], "wb");
    if (!fout || !write_all(fout, status, sizeof status) || !write_all(fout, &total, sizeof total) ||
        !write_all(fout, h_off, sizeof(int32_t) * (size_t)(E + 1)) ||
        !write_all(fout, h_dst, sizeof(int32_t) * n_idx) ||
        !write_all(fout, h_src, sizeof(int32_t) * (size_t)total) ||
        !write_all(fout, h_recv, sizeof(uint16_t) * (size_t)total * H) ||
        !write_all(fout, h_q, (size_t)total * H) ||
        !write_all(fout, h_scales, sizeof(float) * (size_t)total * (H / 128)) ||
        !write_all(fout, h_out, sizeof(uint16_t) * n_x)) {
        fprintf(stderr, "cannot write %s\n", argv[2]);
        return 2;
    }
    fclose(fout);

    ep_handle_destroy(h);
    CK(cudaFree(d_ws));
    CK(cudaFree(d_idx));
    CK(cudaFree(d_x));
    CK(cudaFree(d_w));
    CK(cudaFree(d_y));
    CK(cudaFree(d_out));
    CK(cudaFree(d_recv));
    CK(cudaFree(d_q));
    CK(cudaFree(d_scales));
    CK(cudaStreamDestroy(s));
    free(h_idx);
    free(h_x);
    free(h_w);
    free(h_y);
    free(h_off);
    free(h_dst);
    free(h_out);
    free(h_src);
    free(h_recv);
    free(h_q);
    free(h_scales);
    return rc;
}
