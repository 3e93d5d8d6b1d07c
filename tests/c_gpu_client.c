/*
 * A C client that runs the ZeRO step on the GPU through libzero_b200.so with
 * nothing but the CUDA runtime API: device memory from cudaMalloc, copies
 * with cudaMemcpy, every step of the method in the library. Built and run
 * by tests/test_c_abi_client.py (GPU tests), which checks its output
 * against the oracle.
 *
 *   c_gpu_client in_file out_file
 *
 * in_file (little-endian): int64 n, R, dtype, mode, steps, growth_interval;
 * float init_scale; int64 numels[n]; then, in the plan's padded flat layout
 * of T elements: float master[T]; uint16 param[T]; uint16 grads[steps][R][T].
 * The steps run fused with ping-pong state (zero_step with the replicas).
 * out_file: float scale; int32 cur; int64 good, t; int32 last_overflow,
 * last_skipped; double grad_norm_sq; then the current set's float master[T],
 * m[T], v[T] and uint16 param[T].
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "zero_b200.h"

#define CK(call)                                                                      \
    do {                                                                              \
        cudaError_t e_ = (call);                                                      \
        if (e_ != cudaSuccess) {                                                      \
            fprintf(stderr, "%s:%d: %s\n", __FILE__, __LINE__, cudaGetErrorString(e_)); \
            return 1;                                                                 \
        }                                                                             \
    } while (0)

#define ZK(call)                                                                      \
    do {                                                                              \
        zero_status s_ = (call);                                                      \
        if (s_ != ZERO_OK) {                                                          \
            char m_[512];                                                             \
            zero_last_error(m_, sizeof m_);                                           \
            fprintf(stderr, "%s:%d: status %d: %s\n", __FILE__, __LINE__, (int)s_, m_); \
            return 1;                                                                 \
        }                                                                             \
    } while (0)

static int rd(FILE* f, void* p, size_t n) { return fread(p, 1, n, f) == n ? 0 : 1; }

int main(int argc, char** argv) {
    if (argc != 3) return 2;
    FILE* in = fopen(argv[1], "rb");
    if (!in) return 2;
    int64_t hdr[6];
    float init_scale;
    if (rd(in, hdr, sizeof hdr) || rd(in, &init_scale, sizeof init_scale)) return 2;
    const int64_t n = hdr[0], steps = hdr[4];
    const int32_t R = (int32_t)hdr[1], dtype = (int32_t)hdr[2], mode = (int32_t)hdr[3];
    int64_t* numels = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
    if (!numels || rd(in, numels, sizeof(int64_t) * (size_t)n)) return 2;

    zero_plan_config pc;
    memset(&pc, 0, sizeof pc);
    pc.R = R;
    pc.dtype = dtype;
    pc.tensor_align = 8;
    zero_plan_t* plan = NULL;
    ZK(zero_plan(numels, NULL, n, &pc, &plan));
    zero_plan_info info;
    ZK(zero_plan_get_info(plan, &info));
    const size_t S = (size_t)info.S, T = (size_t)info.T;

    float* h_master = (float*)malloc(sizeof(float) * T);
    uint16_t* h_param = (uint16_t*)malloc(sizeof(uint16_t) * T);
    uint16_t* h_grads = (uint16_t*)malloc(sizeof(uint16_t) * T * (size_t)R);
    if (!h_master || !h_param || !h_grads) return 2;
    if (rd(in, h_master, sizeof(float) * T) || rd(in, h_param, sizeof(uint16_t) * T)) return 2;

    /* two state sets of R shards each, and R full gradient replicas */
    float* master[2][ZERO_MAX_RANKS];
    float* m[2][ZERO_MAX_RANKS];
    float* v[2][ZERO_MAX_RANKS];
    void* param[2][ZERO_MAX_RANKS];
    void* grads[ZERO_MAX_RANKS];
    for (int k = 0; k < 2; k++)
        for (int r = 0; r < R; r++) {
            CK(cudaMalloc((void**)&master[k][r], sizeof(float) * S));
            CK(cudaMalloc((void**)&m[k][r], sizeof(float) * S));
            CK(cudaMalloc((void**)&v[k][r], sizeof(float) * S));
            CK(cudaMalloc(&param[k][r], sizeof(uint16_t) * S));
            CK(cudaMemcpy(master[k][r], h_master + (size_t)r * S, sizeof(float) * S, cudaMemcpyHostToDevice));
            CK(cudaMemcpy(param[k][r], h_param + (size_t)r * S, sizeof(uint16_t) * S, cudaMemcpyHostToDevice));
            CK(cudaMemset(m[k][r], 0, sizeof(float) * S));
            CK(cudaMemset(v[k][r], 0, sizeof(float) * S));
        }
    for (int r = 0; r < R; r++) CK(cudaMalloc(&grads[r], sizeof(uint16_t) * T));

    zero_state st;
    memset(&st, 0, sizeof st);
    for (int k = 0; k < 2; k++) {
        st.master[k] = master[k];
        st.m[k] = m[k];
        st.v[k] = v[k];
        st.param[k] = param[k];
    }
    zero_loss_scale_config lc;
    memset(&lc, 0, sizeof lc);
    lc.mode = mode;
    lc.init_scale = init_scale;
    lc.growth_interval = hdr[5];
    lc.growth_factor = 2.0f;
    lc.backoff_factor = 0.5f;
    lc.min_scale = 1.0f;
    zero_ctx_t* ctx = NULL;
    ZK(zero_ctx_create(plan, &lc, &ctx));
    zero_adamw hp = {1e-3, 0.9, 0.999, 1e-8, 0.01};

    for (int64_t s = 0; s < steps; s++) {
        if (rd(in, h_grads, sizeof(uint16_t) * T * (size_t)R)) return 2;
        for (int r = 0; r < R; r++)
            CK(cudaMemcpy(grads[r], h_grads + (size_t)r * T, sizeof(uint16_t) * T, cudaMemcpyHostToDevice));
        ZK(zero_step(ctx, &hp, &st, (const void* const*)grads, NULL));
    }
    fclose(in);
    ZK(zero_sync(ctx, NULL));
    zero_loss_scale_state ls;
    ZK(zero_loss_scale(ctx, &ls, ZERO_LOSS_SCALE_GET, NULL));

    FILE* out = fopen(argv[2], "wb");
    if (!out) return 2;
    fwrite(&ls.scale, sizeof ls.scale, 1, out);
    fwrite(&ls.cur, sizeof ls.cur, 1, out);
    fwrite(&ls.good, sizeof ls.good, 1, out);
    fwrite(&ls.t, sizeof ls.t, 1, out);
    fwrite(&ls.last_overflow, sizeof ls.last_overflow, 1, out);
    fwrite(&ls.last_skipped, sizeof ls.last_skipped, 1, out);
    fwrite(&ls.grad_norm_sq, sizeof ls.grad_norm_sq, 1, out);
    float* buf = (float*)malloc(sizeof(float) * S);
    if (!buf) return 2;
    const int c = ls.cur;
    float** sets[3] = {master[c], m[c], v[c]};
    for (int f = 0; f < 3; f++)
        for (int r = 0; r < R; r++) {
            CK(cudaMemcpy(buf, sets[f][r], sizeof(float) * S, cudaMemcpyDeviceToHost));
            fwrite(buf, sizeof(float), S, out);
        }
    for (int r = 0; r < R; r++) {
        CK(cudaMemcpy(buf, param[c][r], sizeof(uint16_t) * S, cudaMemcpyDeviceToHost));
        fwrite(buf, sizeof(uint16_t), S, out);
    }
    fclose(out);
    ZK(zero_ctx_destroy(ctx));
    for (int k = 0; k < 2; k++)
        for (int r = 0; r < R; r++) {
            cudaFree(master[k][r]);
            cudaFree(m[k][r]);
            cudaFree(v[k][r]);
            cudaFree(param[k][r]);
        }
    for (int r = 0; r < R; r++) cudaFree(grads[r]);
    zero_plan_destroy(plan);
    free(buf);
    free(h_master);
    free(h_param);
    free(h_grads);
    free(numels);
    return 0;
}
