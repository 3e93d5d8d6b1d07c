/*
 * A plain C99 client of libzero_b200.so, built by tests/test_c_abi_client.py
 * with gcc -std=c99 -pedantic -Werror against include/zero_b200.h. It calls
 * the host-side entry points only (no GPU is needed) and prints what it gets
 * as "key value..." lines for the test to check against the oracle.
 *
 *   c_abi_client plan  R dtype align bucket_elems n numel_0 .. numel_{n-1}
 *       plan, its info, every tensor / bucket / layer range, memory per stage
 *   c_abi_client cpu_step R dtype n numel_0 .. numel_{n-1} in_file out_file
 *       one zero_cpu_step (NONE mode, fixed hyper-parameters) on host shards
 *       read from in_file (acc, master, m, v: R*S fp32 each, rank after rank)
 *       writing out_file (master, m, v as fp32, then param as uint16)
 *   c_abi_client cpu_step_shard ...
 *       the same step one owner at a time (zero_cpu_scan_shard, the summed
 *       totals, zero_cpu_decide, zero_cpu_update_shard, zero_cpu_commit)
 *   c_abi_client errors
 *       error statuses and messages of a few invalid calls
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "zero_b200.h"

static int fail(const char* what, zero_status s) {
    char msg[512];
    zero_last_error(msg, sizeof msg);
    fprintf(stderr, "%s: status %d: %s\n", what, (int)s, msg);
    return 1;
}

static int make_plan(int argc, char** argv, int first, int32_t R, int32_t dtype, int32_t align,
                     int64_t bucket, zero_plan_t** plan, int* next) {
    if (first >= argc) return 2;
    int64_t n = atoll(argv[first]);
    if (n < 1 || first + 1 + n > argc) return 2;
    int64_t* numels = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
    if (!numels) return 2;
    for (int64_t k = 0; k < n; k++) numels[k] = atoll(argv[first + 1 + k]);
    zero_plan_config cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.R = R;
    cfg.dtype = dtype;
    cfg.tensor_align = align;
    cfg.bucket_elems = bucket;
    zero_status s = zero_plan(numels, NULL, n, &cfg, plan);
    free(numels);
    if (s != ZERO_OK) return fail("zero_plan", s);
    *next = first + 1 + (int)n;
    return 0;
}

static int cmd_plan(int argc, char** argv) {
    if (argc < 7) return 2;
    zero_plan_t* plan = NULL;
    int next = 0;
    int rc = make_plan(argc, argv, 6, atoi(argv[2]), atoi(argv[3]), atoi(argv[4]), atoll(argv[5]),
                       &plan, &next);
    if (rc) return rc;
    zero_plan_info info;
    zero_status s = zero_plan_get_info(plan, &info);
    if (s != ZERO_OK) return fail("zero_plan_get_info", s);
    printf("info %lld %lld %lld %lld %lld %lld %lld\n", (long long)info.P, (long long)info.L,
           (long long)info.S, (long long)info.T, (long long)info.n_tensors,
           (long long)info.n_buckets, (long long)info.n_layers);
    for (int64_t k = 0; k < info.n_tensors; k++) {
        int64_t off, numel, bucket, layer;
        if ((s = zero_plan_tensor(plan, k, &off, &numel, &bucket, &layer)) != ZERO_OK)
            return fail("zero_plan_tensor", s);
        printf("tensor %lld %lld %lld %lld\n", (long long)off, (long long)numel, (long long)bucket,
               (long long)layer);
    }
    for (int64_t b = 0; b < info.n_buckets; b++) {
        int64_t lo, hi;
        if ((s = zero_plan_bucket(plan, b, &lo, &hi)) != ZERO_OK) return fail("zero_plan_bucket", s);
        printf("bucket %lld %lld\n", (long long)lo, (long long)hi);
    }
    for (int64_t l = 0; l < info.n_layers; l++) {
        int64_t lo, hi;
        if ((s = zero_plan_layer(plan, l, &lo, &hi)) != ZERO_OK) return fail("zero_plan_layer", s);
        printf("layer %lld %lld\n", (long long)lo, (long long)hi);
    }
    for (int32_t stage = 0; stage <= 3; stage++) {
        int64_t bytes;
        if ((s = zero_plan_memory(plan, stage, &bytes)) != ZERO_OK) return fail("zero_plan_memory", s);
        printf("memory %d %lld\n", (int)stage, (long long)bytes);
    }
    zero_plan_destroy(plan);
    return 0;
}

static int read_all(FILE* f, void* p, size_t bytes) { return fread(p, 1, bytes, f) == bytes ? 0 : 1; }

static int cmd_cpu_step(int argc, char** argv, int sharded) {
    if (argc < 5) return 2;
    int32_t R = atoi(argv[2]), dtype = atoi(argv[3]);
    zero_plan_t* plan = NULL;
    int next = 0;
    int rc = make_plan(argc, argv, 4, R, dtype, 8, 0, &plan, &next);
    if (rc) return rc;
    if (next + 2 > argc) return 2;
    zero_plan_info info;
    zero_plan_get_info(plan, &info);
    const size_t S = (size_t)info.S;
    float* buf = (float*)malloc(sizeof(float) * 4 * (size_t)R * S);
    uint16_t* param = (uint16_t*)calloc((size_t)R * S, sizeof(uint16_t));
    if (!buf || !param) return 2;
    FILE* in = fopen(argv[next], "rb");
    if (!in || read_all(in, buf, sizeof(float) * 4 * (size_t)R * S)) return 2;
    fclose(in);
    const float* acc[ZERO_MAX_RANKS];
    float* master[ZERO_MAX_RANKS];
    float* m[ZERO_MAX_RANKS];
    float* v[ZERO_MAX_RANKS];
    void* par[ZERO_MAX_RANKS];
    for (int r = 0; r < R; r++) {
        acc[r] = buf + (size_t)r * S;
        master[r] = buf + ((size_t)R + r) * S;
        m[r] = buf + (2 * (size_t)R + r) * S;
        v[r] = buf + (3 * (size_t)R + r) * S;
        par[r] = param + (size_t)r * S;
    }
    zero_loss_scale_config cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.mode = ZERO_SCALE_NONE;
    cfg.init_scale = 1.0f;
    zero_loss_scale_state st;
    memset(&st, 0, sizeof st);
    st.scale = 1.0f;
    zero_adamw hp = {1e-3, 0.9, 0.999, 1e-8, 0.01};
    zero_status s = ZERO_OK;
    if (!sharded) {
        s = zero_cpu_step(plan, &cfg, &st, &hp, NULL, acc, master, m, v, par, 2);
        if (s != ZERO_OK) return fail("zero_cpu_step", s);
    } else {
        /* one owner at a time, as separate processes would: its totals, the
           summed totals, one decision, its own update, one commit */
        double total[2] = {0.0, 0.0};
        for (int32_t o = 0; o < R; o++) {
            double part[2];
            s = zero_cpu_scan_shard(plan, &cfg, &st, NULL, acc, o, o + 1, 2, part);
            if (s != ZERO_OK) return fail("zero_cpu_scan_shard", s);
            total[0] += part[0];
            total[1] += part[1];
        }
        zero_cpu_decision d;
        s = zero_cpu_decide(plan, &cfg, &st, NULL, total, &d);
        if (s != ZERO_OK) return fail("zero_cpu_decide", s);
        for (int32_t o = 0; o < R; o++) {
            s = zero_cpu_update_shard(plan, &st, &hp, &d, acc, master, m, v, par, o, o + 1, 2);
            if (s != ZERO_OK) return fail("zero_cpu_update_shard", s);
        }
        s = zero_cpu_commit(&cfg, &st, &d);
        if (s != ZERO_OK) return fail("zero_cpu_commit", s);
    }
    printf("state %lld %d %d %.17g\n", (long long)st.t, (int)st.last_overflow, (int)st.last_skipped,
           st.grad_norm_sq);
    FILE* out = fopen(argv[next + 1], "wb");
    if (!out) return 2;
    fwrite(buf + (size_t)R * S, sizeof(float), 3 * (size_t)R * S, out);
    fwrite(param, sizeof(uint16_t), (size_t)R * S, out);
    fclose(out);
    free(buf);
    free(param);
    zero_plan_destroy(plan);
    return 0;
}

static void report(const char* what, zero_status s) {
    char msg[512];
    size_t n = zero_last_error(msg, sizeof msg);
    printf("error %s %d %zu %s\n", what, (int)s, n, msg);
}

static int cmd_errors(void) {
    zero_plan_config cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.R = 4;
    cfg.dtype = ZERO_BF16;
    cfg.tensor_align = 8;
    int64_t numels[2] = {100, 0};
    zero_plan_t* plan = NULL;
    report("empty_list", zero_plan(numels, NULL, 0, &cfg, &plan));
    report("zero_numel", zero_plan(numels, NULL, 2, &cfg, &plan));
    cfg.R = ZERO_MAX_RANKS + 1;
    report("too_many_ranks", zero_plan(numels, NULL, 1, &cfg, &plan));
    cfg.R = 4;
    cfg.dtype = 7;
    report("bad_dtype", zero_plan(numels, NULL, 1, &cfg, &plan));
    cfg.dtype = ZERO_FP16;
    int32_t layers[2] = {0, 2};
    numels[1] = 5;
    report("layer_gap", zero_plan(numels, layers, 2, &cfg, &plan));
    zero_status s = zero_plan(numels, NULL, 2, &cfg, &plan);
    if (s != ZERO_OK) return fail("zero_plan", s);
    int64_t lo, hi, bytes;
    report("bucket_range", zero_plan_bucket(plan, 99, &lo, &hi));
    report("layer_range", zero_plan_layer(plan, -1, &lo, &hi));
    report("memory_stage", zero_plan_memory(plan, 4, &bytes));
    report("ctx_null", zero_ctx_destroy(NULL));
    zero_plan_destroy(plan);
    printf("version %s\n", zero_version());
    return 0;
}

int main(int argc, char** argv) {
    if (argc < 2) return 2;
    if (strcmp(argv[1], "plan") == 0) return cmd_plan(argc, argv);
    if (strcmp(argv[1], "cpu_step") == 0) return cmd_cpu_step(argc, argv, 0);
    if (strcmp(argv[1], "cpu_step_shard") == 0) return cmd_cpu_step(argc, argv, 1);
    if (strcmp(argv[1], "errors") == 0) return cmd_errors();
    return 2;
}
