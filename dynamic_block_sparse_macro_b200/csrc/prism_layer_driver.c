/*
 * prism_layer_driver: one Prism layer step from C, through the library's C ABI
 * only (include/prism.h, libprism.so), from host buffers.
 *
 *   prism_layer_driver offsets    print sizeof(prism_layer_t) and each field's
 *                                 offset (no CUDA call; a check for bindings)
 *   prism_layer_driver run DIR    read DIR/problem.txt and the raw raster inputs
 *                                 DIR/{Q,K,V,hhat,dO}.bin, run one step with
 *                                 prism_layer_step_host, write DIR/{O,dQ,dK,dV}.bin
 *
 * problem.txt holds: T H W heads head_dim audio_dim dtype(0 f32, 1 bf16)
 * top_k top_p with_backward.  The driver is the caller the library expects: it
 * allocates the device arena and the page-locked host buffers itself.
 */
#include <stddef.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "prism.h"

#define FIELD(f) printf("%s %zu\n", #f, offsetof(prism_layer_t, f))

static int offsets(void) {
    printf("sizeof %zu\n", sizeof(prism_layer_t));
    FIELD(prob); FIELD(top_k); FIELD(top_p); FIELD(eps); FIELD(tau128); FIELD(tau256); FIELD(scale);
    FIELD(guidance); FIELD(fixed_shape); FIELD(with_backward); FIELD(with_io); FIELD(raster);
    FIELD(p_blocks);
    FIELD(g); FIELD(rho); FIELD(abar); FIELD(zone_stats); FIELD(ws_ind); FIELD(ws_ind_bytes);
    FIELD(shape_id); FIELD(perm); FIELD(blk_start); FIELD(gran_blk); FIELD(n_blk); FIELD(margin_shape);
    FIELD(Qp); FIELD(Kp); FIELD(Vp); FIELD(Qbar); FIELD(Kbar); FIELD(P); FIELD(sel); FIELD(gsel);
    FIELD(gselT); FIELD(sel_count); FIELD(margin_sel); FIELD(dev_status); FIELD(Op); FIELD(Of32);
    FIELD(lse); FIELD(ws_fwd); FIELD(ws_fwd_bytes); FIELD(dOp); FIELD(dQp); FIELD(dKp); FIELD(dVp);
    FIELD(ws_bwd); FIELD(ws_bwd_bytes); FIELD(Q); FIELD(K); FIELD(V); FIELD(hhat); FIELD(O); FIELD(dO);
    FIELD(dQ); FIELD(dK); FIELD(dV); FIELD(io_events);
    return 0;
}

static int fail(const char* what, const char* detail) {
    fprintf(stderr, "prism_layer_driver: %s%s%s\n", what, detail ? ": " : "", detail ? detail : "");
    return 1;
}

#define CK(call)                                                                  \
    do {                                                                          \
        cudaError_t e_ = (call);                                                  \
        if (e_ != cudaSuccess) return fail(#call, cudaGetErrorString(e_));        \
    } while (0)
#define PK(call)                                                                  \
    do {                                                                          \
        prism_status_t s_ = (call);                                               \
        if (s_ != PRISM_OK) return fail(#call, prism_status_string(s_));          \
    } while (0)

static int read_file(const char* dir, const char* name, void* dst, size_t bytes) {
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE* f = fopen(path, "rb");
    if (!f) return fail("cannot open", path);
    size_t n = fread(dst, 1, bytes, f);
    fclose(f);
    return n == bytes ? 0 : fail("short read", path);
}

static int write_file(const char* dir, const char* name, const void* src, size_t bytes) {
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE* f = fopen(path, "wb");
    if (!f) return fail("cannot create", path);
    size_t n = fwrite(src, 1, bytes, f);
    fclose(f);
    return n == bytes ? 0 : fail("short write", path);
}

static int run(const char* dir) {
    char path[4096];
    snprintf(path, sizeof path, "%s/problem.txt", dir);
    FILE* f = fopen(path, "r");
    if (!f) return fail("cannot open", path);
    prism_problem_t prob;
    int top_k = 0, with_bwd = 1;
    float top_p = 0.f;
    int got = fscanf(f, "%d %d %d %d %d %d %d %d %f %d", &prob.T, &prob.H, &prob.W, &prob.heads, &prob.head_dim,
                     &prob.audio_dim, &prob.dtype, &top_k, &top_p, &with_bwd);
    fclose(f);
    if (got != 10) return fail("bad problem.txt", path);

    prism_layer_t L;
    PK(prism_layer_init(&L, &prob));
    L.top_k = top_k;
    L.top_p = top_p;
    L.with_backward = with_bwd;
    L.with_io = 1;
    size_t arena_bytes = 0;
    PK(prism_layer_arena_bytes(&L, &arena_bytes));
    void* arena = NULL;
    CK(cudaMalloc(&arena, arena_bytes));
    PK(prism_layer_bind(&L, arena, arena_bytes));
    CK(cudaMemset(L.dev_status, 0, sizeof(uint32_t)));

    prism_sizes_t s;
    PK(prism_query_sizes(&prob, &s));
    const size_t esz = prob.dtype == PRISM_BF16 ? 2 : 4;
    const size_t tok = (size_t)s.n_tokens * prob.heads * prob.head_dim * esz;
    const size_t hhb = (size_t)s.n_tokens * prob.audio_dim * esz;
    const char* in_names[5] = {"Q.bin", "K.bin", "V.bin", "hhat.bin", "dO.bin"};
    const char* out_names[4] = {"O.bin", "dQ.bin", "dK.bin", "dV.bin"};
    void* hin[5] = {0};
    void* hout[4] = {0};
    for (int i = 0; i < 5; ++i) {
        if (i == 4 && !with_bwd) break;
        const size_t b = i == 3 ? hhb : tok;
        CK(cudaMallocHost(&hin[i], b));
        if (read_file(dir, in_names[i], hin[i], b)) return 1;
    }
    for (int i = 0; i < (with_bwd ? 4 : 1); ++i) CK(cudaMallocHost(&hout[i], tok));

    cudaStream_t compute, h2d, d2h;
    CK(cudaStreamCreateWithFlags(&compute, cudaStreamNonBlocking));
    CK(cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking));
    CK(cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking));
    PK(prism_layer_step_host(&L, hin[0], hin[1], hin[2], hin[3], hin[4], hout[0], hout[1], hout[2], hout[3], compute,
                             h2d, d2h));
    CK(cudaStreamSynchronize(d2h));
    uint32_t st = 0;
    PK(prism_read_status(L.dev_status, &st, compute));
    printf("dev_status %u\n", st);
    for (int i = 0; i < (with_bwd ? 4 : 1); ++i)
        if (write_file(dir, out_names[i], hout[i], tok)) return 1;
    for (int i = 0; i < 5; ++i) if (hin[i]) cudaFreeHost(hin[i]);
    for (int i = 0; i < 4; ++i) if (hout[i]) cudaFreeHost(hout[i]);
    cudaStreamDestroy(compute);
    cudaStreamDestroy(h2d);
    cudaStreamDestroy(d2h);
    PK(prism_layer_release(&L));
    cudaFree(arena);
    return st == 0 ? 0 : 2;
}

int main(int argc, char** argv) {
    if (argc >= 2 && strcmp(argv[1], "offsets") == 0) return offsets();
    if (argc >= 3 && strcmp(argv[1], "run") == 0) return run(argv[2]);
    fprintf(stderr, "usage: %s offsets | run DIR\n", argv[0]);
    return 64;
}
