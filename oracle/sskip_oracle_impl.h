/*
 * Body of the CPU oracle, included twice by sskip_oracle.c: once with
 * REAL = float (suffix _f32, the precision the method's spec fixes for its
 * oracle) and once with REAL = double (suffix _f64).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this code.
 *
 * The algorithm follows the TensorRT-LLM Skip-Softmax article
 * ("Skip Softmax 的三步走算法" section): per attention block, take the
 * block's local maximum logit, compare it with the running global maximum,
 * and when the gap exceeds the threshold skip the block's softmax, its second
 * matmul (P.V) and the V block.  The threshold is threshold_scale_factor / L
 * ("实战演练" section: the factor is divided by the context length).
 *
 * The carrier is the plain FlashAttention online softmax (same article,
 * "Skip Softmax 到底怎么回事" section): logits -> running max and sum -> P.V.
 *
 * Readings the pages leave open, fixed here (and matched by the GPU path):
 *   - logits are scaled by sm_scale; natural exp / natural log;
 *   - a row passes when (m_local - m_run) < ln t, strictly; ln 0 = -inf;
 *     a row with m_local = -inf passes iff t > 0; a row with m_run = -inf
 *     and finite m_local fails;
 *   - a block is skipped only when every valid row passes; padding rows
 *     (index >= L) do not vote;
 *   - optional finer vote (SpargeAttn article, "稀疏 Warp 在线 Softmax"
 *     stage: the same local-vs-global maximum test taken per warp): the Br
 *     rows of a query tile are cut into slices of vote_rows rows, each
 *     slice votes alone with the same rule and a slice that passes leaves
 *     its rows' m, l and O untouched; the block (its V and P.V) is skipped
 *     only when every slice passes.  vote_rows = Br is the block vote;
 *   - key blocks are visited in ascending order; m_run is the state before
 *     the block; a skipped block leaves m, l and O untouched;
 *   - prefill: a block is Br rows of ONE query head; query head hq reads kv
 *     head hq / (Hq / Hkv); t = tsf / L of the call;
 *   - decode: a block is the G = Hq/Hkv query heads of one kv head over Bc
 *     keys (one joint vote); t = tsf / seqlens[b]; split s covers key tiles
 *     [s*c, min((s+1)*c, n_k)) with c = ceil(n_k / num_splits), each split
 *     starting from m_run = -inf; an empty split has lse = -inf, O = 0;
 *     the splits merge by log-sum-exp.
 */

#define CAT_(a, b) a##b
#define CAT(a, b) CAT_(a, b)
#define FN(name) CAT(name, SUFFIX)

/* ------------------------------------------------------------------ */
/* Row pass rule: exp(m_local - m_run) < t written in the log domain.   */
/* ------------------------------------------------------------------ */
static int FN(row_passes)(REAL m_local, REAL m_run, REAL ln_t, int t_positive) {
    if (m_local == -(REAL)INFINITY) return t_positive;
    if (m_run == -(REAL)INFINITY) return 0;
    return (m_local - m_run) < ln_t;
}

/* Margin of one row: ln t - (m_local - m_run); the block is skipped iff the
 * minimum margin over valid rows is > 0 (up to the strict/non-strict tie). */
static REAL FN(row_margin)(REAL m_local, REAL m_run, REAL ln_t, int t_positive) {
    if (m_local == -(REAL)INFINITY) return t_positive ? (REAL)INFINITY : -(REAL)INFINITY;
    if (m_run == -(REAL)INFINITY) return -(REAL)INFINITY;
    return ln_t - (m_local - m_run);
}

static REAL FN(dot)(const REAL* a, const REAL* b, int d) {
    REAL s = 0;
    for (int x = 0; x < d; ++x) s += a[x] * b[x];
    return s;
}

/* ------------------------------------------------------------------ */
/* Prefill                                                              */
/* ------------------------------------------------------------------ */
typedef struct {
    const uint16_t *q, *k, *v;
    int B, Hq, Hkv, L, d, causal, Br, Bc, vote_rows;
    REAL scale, ln_t;
    int t_positive;
    const int32_t* units; /* (b, hq, i) triples or NULL = natural order */
    int n_units;
    REAL *o, *lse;        /* [n_units][Br][d], [n_units][Br] */
    int8_t* tile_state;   /* [n_units][n_k] or NULL */
    uint8_t* slice_mask;  /* [n_units][n_k] or NULL: 0 unvisited, else 0x80 | skipped slices */
    REAL* tile_margin;    /* [n_units][n_k] or NULL */
    int64_t skipped, visited, sl_skipped, sl_visited;
    int next;             /* work counter */
    pthread_mutex_t mu;
} FN(prefill_job);

static void FN(prefill_unit)(FN(prefill_job)* J, int u, REAL* qf, REAL* kf, REAL* vf,
                             REAL* S, REAL* m_run, REAL* l, REAL* m_loc,
                             int64_t* cnt /* skipped, visited, slices skipped, slices visited */) {
    const int d = J->d, Br = J->Br, Bc = J->Bc, L = J->L;
    const int R = J->vote_rows, n_sl = Br / R;
    const int n_q = (L + Br - 1) / Br, n_k = (L + Bc - 1) / Bc;
    int b, hq, i;
    if (J->units) {
        b = J->units[3 * u]; hq = J->units[3 * u + 1]; i = J->units[3 * u + 2];
    } else {
        i = u % n_q; hq = (u / n_q) % J->Hq; b = u / (n_q * J->Hq);
    }
    const int G = J->Hq / J->Hkv, kvh = hq / G;
    const int row0 = i * Br;
    const int rows = (L - row0) < Br ? (L - row0) : Br;
    const uint16_t* qp = J->q + (((size_t)b * J->Hq + hq) * L + row0) * d;
    const uint16_t* kp = J->k + ((size_t)b * J->Hkv + kvh) * (size_t)L * d;
    const uint16_t* vp = J->v + ((size_t)b * J->Hkv + kvh) * (size_t)L * d;
    REAL* O = J->o + (size_t)u * Br * d;
    REAL* lse = J->lse + (size_t)u * Br;

    for (int r = 0; r < rows * d; ++r) qf[r] = (REAL)bf16_to_float(qp[r]);
    for (int r = 0; r < Br; ++r) { m_run[r] = -(REAL)INFINITY; l[r] = 0; }
    memset(O, 0, sizeof(REAL) * (size_t)Br * d);

    int j_max = n_k - 1;
    if (J->causal) {
        int jm = ((i + 1) * Br - 1) / Bc;
        if (jm < j_max) j_max = jm;
    }
    if (J->tile_state)
        for (int j = 0; j < n_k; ++j) J->tile_state[(size_t)u * n_k + j] = 0;
    if (J->slice_mask)
        for (int j = 0; j < n_k; ++j) J->slice_mask[(size_t)u * n_k + j] = 0;

    for (int j = 0; j <= j_max; ++j) {
        const int key0 = j * Bc;
        const int keys = (L - key0) < Bc ? (L - key0) : Bc;
        for (int c = 0; c < keys * d; ++c) kf[c] = (REAL)bf16_to_float(kp[(size_t)key0 * d + c]);

        /* Step 1: logits and the block's local row maxima. */
        for (int r = 0; r < rows; ++r) {
            REAL mx = -(REAL)INFINITY;
            for (int c = 0; c < Bc; ++c) {
                REAL s;
                if (c >= keys || (J->causal && key0 + c > row0 + r)) s = -(REAL)INFINITY;
                else s = J->scale * FN(dot)(qf + (size_t)r * d, kf + (size_t)c * d, d);
                S[(size_t)r * Bc + c] = s;
                if (s > mx) mx = s;
            }
            m_loc[r] = mx;
        }

        /* Step 2: compare with the running maximum; every valid row votes,
         * and each slice of R rows decides for itself.  A slice without a
         * valid row passes vacuously and is not counted. */
        int skip = 1;
        unsigned sl_pass = 0;
        REAL margin = (REAL)INFINITY;
        for (int sl = 0; sl < n_sl; ++sl) {
            int pass = 1;
            for (int r = sl * R; r < (sl + 1) * R && r < rows; ++r) {
                if (!FN(row_passes)(m_loc[r], m_run[r], J->ln_t, J->t_positive)) pass = 0;
                REAL mg = FN(row_margin)(m_loc[r], m_run[r], J->ln_t, J->t_positive);
                if (mg < margin) margin = mg;
            }
            if (pass) sl_pass |= 1u << sl;
            else skip = 0;
            if (sl * R < rows) { cnt[3] += 1; cnt[2] += pass; }
        }
        cnt[1] += 1;
        if (J->tile_state) J->tile_state[(size_t)u * n_k + j] = skip ? 2 : 1;
        if (J->slice_mask) J->slice_mask[(size_t)u * n_k + j] = (uint8_t)(0x80u | sl_pass);
        if (J->tile_margin) J->tile_margin[(size_t)u * n_k + j] = margin;

        /* Step 3: a skipped block costs no softmax, no P.V and no V block. */
        if (skip) { cnt[0] += 1; continue; }

        for (int c = 0; c < keys * d; ++c) vf[c] = (REAL)bf16_to_float(vp[(size_t)key0 * d + c]);
        for (int r = 0; r < rows; ++r) {
            if (sl_pass >> (r / R) & 1u) continue; /* this row's slice skipped the block */
            REAL m_new = m_loc[r] > m_run[r] ? m_loc[r] : m_run[r];
            if (m_new == -(REAL)INFINITY) continue; /* nothing visible yet */
            REAL alpha = (m_run[r] == -(REAL)INFINITY) ? 0 : EXP(m_run[r] - m_new);
            REAL* Or = O + (size_t)r * d;
            l[r] *= alpha;
            for (int x = 0; x < d; ++x) Or[x] *= alpha;
            for (int c = 0; c < keys; ++c) {
                REAL s = S[(size_t)r * Bc + c];
                if (s == -(REAL)INFINITY) continue;
                REAL p = EXP(s - m_new);
                l[r] += p;
                const REAL* vr = vf + (size_t)c * d;
                for (int x = 0; x < d; ++x) Or[x] += p * vr[x];
            }
            m_run[r] = m_new;
        }
    }

    /* Epilogue: normalise and form the log-sum-exp of the kept keys. */
    for (int r = 0; r < Br; ++r) {
        REAL* Or = O + (size_t)r * d;
        if (r >= rows || l[r] == 0) {
            for (int x = 0; x < d; ++x) Or[x] = 0;
            lse[r] = -(REAL)INFINITY;
            continue;
        }
        for (int x = 0; x < d; ++x) Or[x] = Or[x] / l[r];
        lse[r] = m_run[r] + LOG(l[r]);
    }
}

static void* FN(prefill_worker)(void* arg) {
    FN(prefill_job)* J = (FN(prefill_job)*)arg;
    const int d = J->d, Br = J->Br, Bc = J->Bc;
    REAL* qf = (REAL*)malloc(sizeof(REAL) * (size_t)Br * d);
    REAL* kf = (REAL*)malloc(sizeof(REAL) * (size_t)Bc * d);
    REAL* vf = (REAL*)malloc(sizeof(REAL) * (size_t)Bc * d);
    REAL* S = (REAL*)malloc(sizeof(REAL) * (size_t)Br * Bc);
    REAL* m_run = (REAL*)malloc(sizeof(REAL) * Br);
    REAL* l = (REAL*)malloc(sizeof(REAL) * Br);
    REAL* m_loc = (REAL*)malloc(sizeof(REAL) * Br);
    int64_t cnt[4] = {0, 0, 0, 0};
    for (;;) {
        int u = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (u >= J->n_units) break;
        FN(prefill_unit)(J, u, qf, kf, vf, S, m_run, l, m_loc, cnt);
    }
    pthread_mutex_lock(&J->mu);
    J->skipped += cnt[0];
    J->visited += cnt[1];
    J->sl_skipped += cnt[2];
    J->sl_visited += cnt[3];
    pthread_mutex_unlock(&J->mu);
    free(qf); free(kf); free(vf); free(S); free(m_run); free(l); free(m_loc);
    return NULL;
}

int FN(sskip_oracle_prefill)(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             int B, int Hq, int Hkv, int L, int d, int causal,
                             double sm_scale, double threshold_scale_factor, int Br, int Bc,
                             int vote_rows, const int32_t* units, int n_units,
                             REAL* o, REAL* lse, int64_t* counts /* [4] */,
                             int8_t* tile_state, uint8_t* slice_mask, REAL* tile_margin,
                             int nthreads) {
    if (!q || !k || !v || !o || !lse || !counts) return 1;
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || L < 1 || d < 1 || Br < 1 || Bc < 1) return 1;
    if (vote_rows < 1 || vote_rows > Br || Br % vote_rows || Br / vote_rows > 7) return 1;
    if (!(threshold_scale_factor >= 0)) return 1;
    FN(prefill_job) J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.L = L; J.d = d; J.causal = causal; J.Br = Br; J.Bc = Bc;
    J.vote_rows = vote_rows;
    J.scale = (REAL)sm_scale;
    /* t = threshold_scale_factor / L; compare in the log domain. */
    J.t_positive = threshold_scale_factor > 0;
    J.ln_t = J.t_positive ? (REAL)log(threshold_scale_factor / (double)L) : -(REAL)INFINITY;
    J.units = units;
    J.n_units = units ? n_units : B * Hq * ((L + Br - 1) / Br);
    J.o = o; J.lse = lse; J.tile_state = tile_state; J.slice_mask = slice_mask;
    J.tile_margin = tile_margin;
    pthread_mutex_init(&J.mu, NULL);
    run_workers(FN(prefill_worker), &J, nthreads, J.n_units);
    pthread_mutex_destroy(&J.mu);
    counts[0] = J.skipped;
    counts[1] = J.visited;
    counts[2] = J.sl_skipped;
    counts[3] = J.sl_visited;
    return 0;
}

/* ------------------------------------------------------------------ */
/* Decode: split-KV over the cache of each (batch, kv head), then merge  */
/* ------------------------------------------------------------------ */
typedef struct {
    const uint16_t *q, *kc, *vc;
    const int32_t* seqlens;
    int B, Hq, Hkv, Lmax, d, Bc, S;
    REAL scale;
    double tsf;
    REAL *o, *lse;          /* [B][Hq][d], [B][Hq] */
    REAL *o_part, *lse_part; /* [B][Hq][S][d], [B][Hq][S] or NULL */
    int8_t* tile_state;      /* [B][Hkv][n_k_max] or NULL */
    REAL* tile_margin;
    int n_k_max;
    int64_t skipped, visited;
    int next;
    pthread_mutex_t mu;
} FN(decode_job);

static void FN(decode_group)(FN(decode_job)* J, int unit, REAL* qf, REAL* kf, REAL* vf,
                             REAL* Sm, REAL* m_run, REAL* l, REAL* m_loc, REAL* Oacc,
                             REAL* Op, REAL* lp, int64_t* skipped, int64_t* visited) {
    const int d = J->d, Bc = J->Bc, NS = J->S;
    const int G = J->Hq / J->Hkv;
    const int b = unit / J->Hkv, kvh = unit % J->Hkv;
    const int Lb = J->seqlens[b];
    const int n_k = (Lb + Bc - 1) / Bc;
    const int c_per = (n_k + NS - 1) / NS;
    const int t_positive = J->tsf > 0;
    const REAL ln_t = t_positive ? (REAL)log(J->tsf / (double)Lb) : -(REAL)INFINITY;
    const uint16_t* kp = J->kc + ((size_t)b * J->Hkv + kvh) * (size_t)J->Lmax * d;
    const uint16_t* vp = J->vc + ((size_t)b * J->Hkv + kvh) * (size_t)J->Lmax * d;

    for (int g = 0; g < G; ++g)
        for (int x = 0; x < d; ++x)
            qf[(size_t)g * d + x] = (REAL)bf16_to_float(J->q[(((size_t)b * J->Hq) + kvh * G + g) * d + x]);
    if (J->tile_state)
        for (int j = 0; j < J->n_k_max; ++j) J->tile_state[(size_t)unit * J->n_k_max + j] = 0;

    for (int s = 0; s < NS; ++s) {
        int j0 = s * c_per, j1 = (s + 1) * c_per;
        if (j1 > n_k) j1 = n_k;
        for (int g = 0; g < G; ++g) { m_run[g] = -(REAL)INFINITY; l[g] = 0; }
        memset(Oacc, 0, sizeof(REAL) * (size_t)G * d);
        for (int j = j0; j < j1; ++j) {
            const int key0 = j * Bc;
            const int keys = (Lb - key0) < Bc ? (Lb - key0) : Bc;
            for (int c = 0; c < keys * d; ++c) kf[c] = (REAL)bf16_to_float(kp[(size_t)key0 * d + c]);
            for (int g = 0; g < G; ++g) {
                REAL mx = -(REAL)INFINITY;
                for (int c = 0; c < Bc; ++c) {
                    REAL sc = (c < keys) ? J->scale * FN(dot)(qf + (size_t)g * d, kf + (size_t)c * d, d)
                                         : -(REAL)INFINITY;
                    Sm[(size_t)g * Bc + c] = sc;
                    if (sc > mx) mx = sc;
                }
                m_loc[g] = mx;
            }
            int skip = 1;
            REAL margin = (REAL)INFINITY;
            for (int g = 0; g < G; ++g) {
                if (!FN(row_passes)(m_loc[g], m_run[g], ln_t, t_positive)) skip = 0;
                REAL mg = FN(row_margin)(m_loc[g], m_run[g], ln_t, t_positive);
                if (mg < margin) margin = mg;
            }
            *visited += 1;
            if (J->tile_state) J->tile_state[(size_t)unit * J->n_k_max + j] = skip ? 2 : 1;
            if (J->tile_margin) J->tile_margin[(size_t)unit * J->n_k_max + j] = margin;
            if (skip) { *skipped += 1; continue; }

            for (int c = 0; c < keys * d; ++c) vf[c] = (REAL)bf16_to_float(vp[(size_t)key0 * d + c]);
            for (int g = 0; g < G; ++g) {
                REAL m_new = m_loc[g] > m_run[g] ? m_loc[g] : m_run[g];
                REAL alpha = (m_run[g] == -(REAL)INFINITY) ? 0 : EXP(m_run[g] - m_new);
                REAL* Og = Oacc + (size_t)g * d;
                l[g] *= alpha;
                for (int x = 0; x < d; ++x) Og[x] *= alpha;
                for (int c = 0; c < keys; ++c) {
                    REAL p = EXP(Sm[(size_t)g * Bc + c] - m_new);
                    l[g] += p;
                    const REAL* vr = vf + (size_t)c * d;
                    for (int x = 0; x < d; ++x) Og[x] += p * vr[x];
                }
                m_run[g] = m_new;
            }
        }
        /* The split's normalised partial and its log-sum-exp. */
        for (int g = 0; g < G; ++g) {
            REAL* dst = Op + ((size_t)g * NS + s) * d;
            if (l[g] == 0) {
                for (int x = 0; x < d; ++x) dst[x] = 0;
                lp[(size_t)g * NS + s] = -(REAL)INFINITY;
            } else {
                for (int x = 0; x < d; ++x) dst[x] = Oacc[(size_t)g * d + x] / l[g];
                lp[(size_t)g * NS + s] = m_run[g] + LOG(l[g]);
            }
        }
    }

    /* Merge the splits: lse = log sum_s exp(lse_s); O = sum_s exp(lse_s - lse) O_s. */
    for (int g = 0; g < G; ++g) {
        const int hq = kvh * G + g;
        REAL mx = -(REAL)INFINITY;
        for (int s = 0; s < NS; ++s) if (lp[(size_t)g * NS + s] > mx) mx = lp[(size_t)g * NS + s];
        REAL sum = 0;
        for (int s = 0; s < NS; ++s) {
            REAL ls = lp[(size_t)g * NS + s];
            if (ls != -(REAL)INFINITY) sum += EXP(ls - mx);
        }
        REAL lse_all = mx + LOG(sum);
        REAL* dst = J->o + ((size_t)b * J->Hq + hq) * d;
        for (int x = 0; x < d; ++x) dst[x] = 0;
        for (int s = 0; s < NS; ++s) {
            REAL ls = lp[(size_t)g * NS + s];
            if (ls == -(REAL)INFINITY) continue;
            REAL w = EXP(ls - lse_all);
            for (int x = 0; x < d; ++x) dst[x] += w * Op[((size_t)g * NS + s) * d + x];
        }
        J->lse[(size_t)b * J->Hq + hq] = lse_all;
        if (J->o_part) {
            for (int s = 0; s < NS; ++s) {
                J->lse_part[((size_t)b * J->Hq + hq) * NS + s] = lp[(size_t)g * NS + s];
                for (int x = 0; x < d; ++x)
                    J->o_part[(((size_t)b * J->Hq + hq) * NS + s) * d + x] = Op[((size_t)g * NS + s) * d + x];
            }
        }
    }
}

static void* FN(decode_worker)(void* arg) {
    FN(decode_job)* J = (FN(decode_job)*)arg;
    const int d = J->d, Bc = J->Bc, G = J->Hq / J->Hkv, NS = J->S;
    REAL* qf = (REAL*)malloc(sizeof(REAL) * (size_t)G * d);
    REAL* kf = (REAL*)malloc(sizeof(REAL) * (size_t)Bc * d);
    REAL* vf = (REAL*)malloc(sizeof(REAL) * (size_t)Bc * d);
    REAL* Sm = (REAL*)malloc(sizeof(REAL) * (size_t)G * Bc);
    REAL* m_run = (REAL*)malloc(sizeof(REAL) * G);
    REAL* l = (REAL*)malloc(sizeof(REAL) * G);
    REAL* m_loc = (REAL*)malloc(sizeof(REAL) * G);
    REAL* Oacc = (REAL*)malloc(sizeof(REAL) * (size_t)G * d);
    REAL* Op = (REAL*)malloc(sizeof(REAL) * (size_t)G * NS * d);
    REAL* lp = (REAL*)malloc(sizeof(REAL) * (size_t)G * NS);
    int64_t skipped = 0, visited = 0;
    for (;;) {
        int u = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (u >= J->B * J->Hkv) break;
        FN(decode_group)(J, u, qf, kf, vf, Sm, m_run, l, m_loc, Oacc, Op, lp, &skipped, &visited);
    }
    pthread_mutex_lock(&J->mu);
    J->skipped += skipped;
    J->visited += visited;
    pthread_mutex_unlock(&J->mu);
    free(qf); free(kf); free(vf); free(Sm); free(m_run); free(l); free(m_loc);
    free(Oacc); free(Op); free(lp);
    return NULL;
}

int FN(sskip_oracle_decode)(const uint16_t* q, const uint16_t* kcache, const uint16_t* vcache,
                            const int32_t* seqlens, int B, int Hq, int Hkv, int Lmax, int d,
                            double sm_scale, double threshold_scale_factor, int Bc, int num_splits,
                            REAL* o, REAL* lse, REAL* o_part, REAL* lse_part, int64_t* counts,
                            int8_t* tile_state, REAL* tile_margin, int nthreads) {
    if (!q || !kcache || !vcache || !seqlens || !o || !lse || !counts) return 1;
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || Lmax < 1 || d < 1 || Bc < 1 || num_splits < 1) return 1;
    if (!(threshold_scale_factor >= 0)) return 1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 1 || seqlens[b] > Lmax) return 1;
    if ((o_part == NULL) != (lse_part == NULL)) return 1;
    FN(decode_job) J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.kc = kcache; J.vc = vcache; J.seqlens = seqlens;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.Lmax = Lmax; J.d = d; J.Bc = Bc; J.S = num_splits;
    J.scale = (REAL)sm_scale;
    J.tsf = threshold_scale_factor;
    J.o = o; J.lse = lse; J.o_part = o_part; J.lse_part = lse_part;
    J.tile_state = tile_state; J.tile_margin = tile_margin;
    J.n_k_max = (Lmax + Bc - 1) / Bc;
    pthread_mutex_init(&J.mu, NULL);
    run_workers(FN(decode_worker), &J, nthreads, B * Hkv);
    pthread_mutex_destroy(&J.mu);
    counts[0] = J.skipped;
    counts[1] = J.visited;
    return 0;
}

#undef FN
#undef CAT
#undef CAT_
