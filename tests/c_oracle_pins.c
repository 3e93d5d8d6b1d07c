/*
 * The oracle's pins from C: a strict C99 program that links the oracle
 * (liboracle.so, test infrastructure) and checks it against the stored
 * golden fixtures, with no Python in between. Built and run by
 * tests/test_oracle_c_pins.py.
 *
 *   c_oracle_pins adamw_one_param.txt memory_pages.txt fsm_sequences.txt layout_worked.txt
 *
 * - adamw_one_param.txt: two AdamW steps of one parameter, computed by hand
 *   in exact decimal arithmetic; the oracle's fp32 state must agree to a
 *   few fp32 ulps (the fixture is exact, the oracle rounds every operation).
 * - memory_pages.txt: the per-rank model-state bytes of the pages' worked
 *   figures (~ within 1 %, "over" and "under" as stated).
 * - fsm_sequences.txt: loss-scale state machine sequences written by hand;
 *   every listed step's overflow, skip, scale, clean count and t.
 * - layout_worked.txt: flat layouts worked by hand (offsets, P, L, S, T).
 * Prints one line per failed check and exits non-zero if any failed.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "zero_oracle.h"

static int failures = 0;

static void fail(const char* what, const char* detail) {
    fprintf(stderr, "FAIL %s: %s\n", what, detail);
    failures += 1;
}

static int is_comment_or_blank(const char* line) {
    while (*line == ' ' || *line == '\t') line++;
    return *line == '#' || *line == '\n' || *line == '\0';
}

static int close_rel(double got, double want, double rel) {
    return fabs(got - want) <= rel * fabs(want);
}

static void check_adamw(const char* path) {
    FILE* f = fopen(path, "r");
    if (!f) {
        fail("adamw", "cannot open the fixture");
        return;
    }
    /* p0 = 1, m0 = v0 = 0, g = 0.5 at every step, one rank, bf16 (0.5 is exact) */
    float master = 1.0f, m = 0.0f, v = 0.0f;
    uint16_t param = oracle_float_to_half(1.0f, ORACLE_BF16);
    const uint16_t g = oracle_float_to_half(0.5f, ORACLE_BF16);
    oracle_adamw hp = {1e-3, 0.9, 0.999, 1e-8, 0.01};
    oracle_fsm st;
    memset(&st, 0, sizeof st);
    st.mode = ORACLE_SCALE_NONE;
    st.scale = 1.0f;
    st.growth_interval = 1000;
    st.growth_factor = 2.0f;
    st.backoff_factor = 0.5f;
    st.min_scale = 1.0f;
    char line[512];
    int rows = 0, done = 0;
    while (fgets(line, sizeof line, f)) {
        if (is_comment_or_blank(line)) continue;
        int step;
        double p_want, m_want, v_want;
        if (sscanf(line, "%d %lf %lf %lf", &step, &p_want, &m_want, &v_want) != 4) {
            fail("adamw", "unreadable row");
            continue;
        }
        while (done < step) {
            if (oracle_step(1, 1, ORACLE_BF16, &g, &master, &m, &v, &param, &hp, &st) != 0)
                fail("adamw", "a NONE-mode step was skipped");
            done += 1;
        }
        char msg[256];
        /* a few fp32 ulps of relative agreement with the exact values */
        if (!close_rel(master, p_want, 4e-7) || !close_rel(m, m_want, 4e-7) || !close_rel(v, v_want, 4e-7)) {
            snprintf(msg, sizeof msg, "step %d: p %.11g m %.11g v %.11g", step, (double)master, (double)m,
                     (double)v);
            fail("adamw", msg);
        }
        if (st.t != step) fail("adamw", "step count");
        rows += 1;
    }
    fclose(f);
    if (rows < 2) fail("adamw", "fewer than two rows");
}

static void check_memory(const char* path) {
    FILE* f = fopen(path, "r");
    if (!f) {
        fail("memory", "cannot open the fixture");
        return;
    }
    char line[1024];
    int rows = 0;
    while (fgets(line, sizeof line, f)) {
        if (is_comment_or_blank(line)) continue;
        char what[32], rel[32];
        int stage;
        double psi, n, value;
        if (sscanf(line, "%31s %d %lf %lf %31s %lf", what, &stage, &psi, &n, rel, &value) != 6) {
            fail("memory", "unreadable row");
            continue;
        }
        const double bytes = strcmp(what, "fp32w") == 0 ? oracle_fp32_weight_bytes(psi)
                                                        : oracle_model_state_bytes(stage, psi, n);
        int ok = 0;
        if (strcmp(rel, "approx") == 0) ok = fabs(bytes / value - 1.0) <= 0.01;
        else if (strcmp(rel, "gt") == 0) ok = bytes > value;
        else if (strcmp(rel, "lt") == 0) ok = bytes < value;
        if (!ok) {
            char msg[256];
            snprintf(msg, sizeof msg, "%s stage %d psi %g N %g: %g bytes, want %s %g", what, stage, psi, n,
                     bytes, rel, value);
            fail("memory", msg);
        }
        rows += 1;
    }
    fclose(f);
    if (rows < 5) fail("memory", "fewer than five rows");
}

static int parse_list(char* s, int64_t* out, int cap) {
    int n = 0;
    for (char* tok = strtok(s, ","); tok && n < cap; tok = strtok(NULL, ",")) out[n++] = strtoll(tok, NULL, 10);
    return n;
}

static void check_layout(const char* path) {
    FILE* f = fopen(path, "r");
    if (!f) {
        fail("layout", "cannot open the fixture");
        return;
    }
    char line[1024];
    int rows = 0;
    while (fgets(line, sizeof line, f)) {
        if (is_comment_or_blank(line)) continue;
        char name[64], sizes_s[512], offs_s[512];
        int R, align;
        long long P, L, S, T;
        if (sscanf(line, "%63s %d %d %511s %511s %lld %lld %lld %lld", name, &R, &align, sizes_s, offs_s, &P, &L,
                   &S, &T) != 9) {
            fail("layout", "unreadable row");
            continue;
        }
        int64_t sizes[64], want_off[64], off[64], out[6], tb[64], blo[64], bhi[64], llo[64], lhi[64];
        const int n = parse_list(sizes_s, sizes, 64);
        const int no = parse_list(offs_s, want_off, 64);
        if (n < 1 || no != n) {
            fail("layout", "bad size or offset list");
            continue;
        }
        if (oracle_layout(sizes, n, R, align, 0, NULL, off, out, tb, blo, bhi, llo, lhi) != 0) {
            fail("layout", "oracle_layout rejected a worked example");
            continue;
        }
        int ok = out[0] == P && out[1] == L && out[2] == S && out[3] == T;
        for (int k = 0; k < n; k++) ok = ok && off[k] == want_off[k];
        if (!ok) {
            char msg[256];
            snprintf(msg, sizeof msg, "%s: P %lld L %lld S %lld T %lld", name, (long long)out[0], (long long)out[1],
                     (long long)out[2], (long long)out[3]);
            fail("layout", msg);
        }
        rows += 1;
    }
    fclose(f);
    if (rows < 4) fail("layout", "fewer than four rows");
}

static int mode_of(const char* s) {
    if (strcmp(s, "DYNAMIC") == 0) return ORACLE_SCALE_DYNAMIC;
    if (strcmp(s, "STATIC") == 0) return ORACLE_SCALE_STATIC;
    return ORACLE_SCALE_NONE;
}

static void check_fsm(const char* path) {
    FILE* f = fopen(path, "r");
    if (!f) {
        fail("fsm", "cannot open the fixture");
        return;
    }
    char line[1024];
    int seqs = 0, in_seq = 0;
    oracle_fsm st;
    int ovf[64], n_ovf = 0;
    int64_t done = 0;
    char name[64] = "";
    while (fgets(line, sizeof line, f)) {
        if (is_comment_or_blank(line)) continue;
        if (strncmp(line, "seq ", 4) == 0) {
            char mode[32];
            double init, minimum;
            long long interval;
            if (sscanf(line + 4, "%63s %31s %lf %lld %lf", name, mode, &init, &interval, &minimum) != 5) {
                fail("fsm", "unreadable seq line");
                continue;
            }
            memset(&st, 0, sizeof st);
            st.mode = mode_of(mode);
            st.scale = (float)init;
            st.growth_interval = interval;
            st.growth_factor = 2.0f;
            st.backoff_factor = 0.5f;
            st.min_scale = (float)minimum;
            n_ovf = 0;
            done = 0;
            in_seq = 1;
            continue;
        }
        if (strncmp(line, "ovf", 3) == 0) {
            char* p = line + 3;
            char* end;
            for (long x = strtol(p, &end, 10); end != p && n_ovf < 64; x = strtol(p, &end, 10)) {
                ovf[n_ovf++] = (int)x;
                p = end;
            }
            continue;
        }
        if (strncmp(line, "end", 3) == 0) {
            seqs += in_seq;
            in_seq = 0;
            continue;
        }
        long long step, want_ovf, want_skip, want_good, want_t;
        double want_scale;
        if (!in_seq || sscanf(line, "%lld %lld %lld %lf %lld %lld", &step, &want_ovf, &want_skip, &want_scale,
                              &want_good, &want_t) != 6) {
            fail("fsm", "unreadable row");
            continue;
        }
        int skipped = 0;
        while (done < step) {
            done += 1;
            int o = 0;
            for (int i = 0; i < n_ovf; i++) o |= ovf[i] == done;
            skipped = oracle_fsm_update(&st, o);  /* advances t on an applied step */
        }
        if (st.last_overflow != want_ovf || skipped != want_skip || st.last_skipped != want_skip ||
            (double)st.scale != want_scale ||
            st.good != want_good || st.t != want_t) {
            char msg[256];
            snprintf(msg, sizeof msg, "%s step %lld: overflow %d skipped %d scale %g good %lld t %lld", name, step,
                     (int)st.last_overflow, skipped, (double)st.scale, (long long)st.good, (long long)st.t);
            fail("fsm", msg);
        }
    }
    fclose(f);
    if (seqs < 4) fail("fsm", "fewer than four sequences");
}

int main(int argc, char** argv) {
    if (argc != 5) {
        fprintf(stderr, "usage: %s adamw_one_param.txt memory_pages.txt fsm_sequences.txt layout_worked.txt\n",
                argv[0]);
        return 2;
    }
    check_adamw(argv[1]);
    check_memory(argv[2]);
    check_fsm(argv[3]);
    check_layout(argv[4]);
    if (failures) return 1;
    printf("oracle pins ok\n");
    return 0;
}
