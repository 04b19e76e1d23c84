/*
 * oracle.c -- fp64 CPU oracle for exact attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA path, and the CUDA path never
 * calls it.
 *
 * What it computes (pages: "Flash Attention", 14cs17.netlify.app, sections
 * "Standard Attention Memory Analysis" and "Flash Attention Algorithm";
 * xspy.com "FlashAttention and chunked prefill mechanics", section 1):
 *
 *     S = scale * Q K^T,  P = softmax(S) row-wise,  O = P V,
 *     lse_i = log(sum_j exp(S_ij))           (natural log, scaled scores)
 *
 * Standard attention materialises every score row in full; so does
 * oracle_attention() below, one row at a time, in fp64, on bf16 inputs that
 * are widened exactly.  The pages call the tiled method exact, so this plain
 * definition is the result the GPU path must reach up to rounding.
 *
 * Readings of points the pages leave open:
 *   - scale is a parameter (the pages write softmax(QK^T) with no scale);
 *   - causal means key j is allowed for query i iff j <= i, positions counted
 *     inside the row's own sequence;
 *   - grouped-query attention: query head h reads key/value head
 *     h / (Hq / Hkv) (contiguous groups);
 *   - a row whose every key is masked has O = 0 and lse = -inf, following the
 *     -inf guard of the page's streaming softmax, where an empty prefix adds 0;
 *   - packed variable-length batches: sequence s owns tokens
 *     [cu_seqlens[s], cu_seqlens[s+1]); q, o are [Ntot, Hq, d], k, v are
 *     [Ntot, Hkv, d] and lse is [Hq, Ntot].  Dense batches: q, o are
 *     [B, Hq, N, d], k, v are [B, Hkv, N, d] and lse is [B, Hq, N].
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC oracle.c -o liboracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Widen one bf16 bit pattern to fp64.  bf16 is the top half of an IEEE
 * binary32, so the widening is exact. */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Softmax of one vector (xspy.com page, section 3, "standard_softmax";      */
/* the definition the online form must reproduce).                          */
/* Writes p[0..n) and returns lse = m + log(sum exp(x - m)).                 */
/* ------------------------------------------------------------------------ */
double oracle_softmax(const double* x, int64_t n, double* p) {
    double m = -INFINITY;
    for (int64_t i = 0; i < n; ++i)
        if (x[i] > m) m = x[i];
    if (m == -INFINITY) {            /* empty or fully masked row */
        for (int64_t i = 0; i < n; ++i) p[i] = 0.0;
        return -INFINITY;
    }
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        p[i] = exp(x[i] - m);
        s += p[i];
    }
    for (int64_t i = 0; i < n; ++i) p[i] /= s;
    return m + log(s);
}

/* ------------------------------------------------------------------------ */
/* Streaming (online) softmax over blocks, in the two passes of the          */
/* xspy.com page, section 3: pass 1 walks the blocks keeping a running max   */
/* and a running denominator, rescaling the old denominator by               */
/* exp(m_old - m_new) whenever the max grows (the rescale of Theorem 2 on    */
/* the 14cs17 page); pass 2 normalises every element by the final pair.      */
/*                                                                          */
/* x is split into nblocks consecutive blocks of lengths block_len[]; the   */
/* blocks are visited in the order given by order[] (a permutation of       */
/* 0..nblocks-1, or NULL for 0,1,2,...).  Returns lse = m + log(d).          */
/* ------------------------------------------------------------------------ */
double oracle_online_softmax(const double* x, const int64_t* block_len,
                             int64_t nblocks, const int64_t* order, double* p) {
    int64_t* start = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nblocks + 1));
    int64_t n = 0;
    for (int64_t b = 0; b < nblocks; ++b) { start[b] = n; n += block_len[b]; }
    start[nblocks] = n;

    double m_run = -INFINITY;   /* running max over the blocks seen so far */
    double d_run = 0.0;         /* running sum of exp(x - m_run)           */
    for (int64_t t = 0; t < nblocks; ++t) {
        int64_t b = order ? order[t] : t;
        double m_blk = -INFINITY;
        for (int64_t i = start[b]; i < start[b + 1]; ++i)
            if (x[i] > m_blk) m_blk = x[i];
        double m_new = m_run > m_blk ? m_run : m_blk;
        if (m_new == -INFINITY) continue;   /* nothing but -inf so far */
        /* guard: an empty prefix (m_run = -inf) contributes nothing */
        double carry = (m_run == -INFINITY) ? 0.0 : exp(m_run - m_new);
        double blk = 0.0;
        for (int64_t i = start[b]; i < start[b + 1]; ++i) blk += exp(x[i] - m_new);
        d_run = carry * d_run + blk;
        m_run = m_new;
    }
    for (int64_t i = 0; i < n; ++i)
        p[i] = (m_run == -INFINITY) ? 0.0 : exp(x[i] - m_run) / d_run;
    free(start);
    return (m_run == -INFINITY) ? -INFINITY : m_run + log(d_run);
}

/* ------------------------------------------------------------------------ */
/* Layout helpers shared by the two attention functions of this file.        */
/* ------------------------------------------------------------------------ */
typedef struct {
    const uint16_t *q, *k, *v;
    int B, Hq, Hkv, N, d;
    double scale;
    int causal;
    const int32_t* cu;      /* NULL: dense */
} attn_t;

/* A query row is named by a row id: dense (b*Hq + h)*N + t, packed h*Ntot +
 * token.  row_info() turns it into the head, the position t inside its
 * sequence, the sequence length and pointers to the first element of the
 * query row and of key/value position 0 of that sequence and kv head. */
typedef struct {
    int h, hk;
    int64_t t, len;
    const uint16_t *qrow, *k0, *v0;
    int64_t kv_stride;   /* elements between consecutive key positions */
} row_t;

static int row_info(const attn_t* a, int64_t rowid, row_t* r) {
    int group = a->Hq / a->Hkv;
    if (!a->cu) {
        int64_t N = a->N;
        int64_t bh = rowid / N;
        r->t = rowid % N;
        r->h = (int)(bh % a->Hq);
        int64_t b = bh / a->Hq;
        if (b >= a->B) return -1;
        r->hk = r->h / group;
        r->len = N;
        r->qrow = a->q + ((b * a->Hq + r->h) * N + r->t) * a->d;
        r->k0 = a->k + ((b * a->Hkv + r->hk) * N) * a->d;
        r->v0 = a->v + ((b * a->Hkv + r->hk) * N) * a->d;
        r->kv_stride = a->d;
    } else {
        int64_t Ntot = a->N;
        r->h = (int)(rowid / Ntot);
        int64_t tok = rowid % Ntot;
        if (r->h >= a->Hq) return -1;
        int s = 0;
        while (s < a->B && !(a->cu[s] <= tok && tok < a->cu[s + 1])) ++s;
        if (s == a->B) return -1;
        r->hk = r->h / group;
        r->t = tok - a->cu[s];
        r->len = a->cu[s + 1] - a->cu[s];
        r->qrow = a->q + (tok * a->Hq + r->h) * a->d;
        r->k0 = a->k + ((int64_t)a->cu[s] * a->Hkv + r->hk) * a->d;
        r->v0 = a->v + ((int64_t)a->cu[s] * a->Hkv + r->hk) * a->d;
        r->kv_stride = (int64_t)a->Hkv * a->d;
    }
    return 0;
}

static int key_allowed(const attn_t* a, const row_t* r, int64_t j) {
    return !a->causal || j <= r->t;
}

/* ------------------------------------------------------------------------ */
/* Standard (materialised) attention, one query row at a time.               */
/* 14cs17 page, "Standard Attention Memory Analysis": S = QK^T, softmax of   */
/* S, O = softmax(S) V -- here with the whole score row held in fp64.        */
/*                                                                          */
/* rows: list of nrows row ids, or NULL for every row (nrows is then        */
/* ignored and the output is indexed by row id).  o: nrows x d, lse: nrows. */
/* Returns 0, or -1 on a row id out of range.                               */
/* ------------------------------------------------------------------------ */
int oracle_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     int B, int Hq, int Hkv, int N, int d, double scale,
                     int causal, const int32_t* cu_seqlens,
                     const int64_t* rows, int64_t nrows,
                     double* o, double* lse, int nthreads) {
    attn_t a = {q, k, v, B, Hq, Hkv, N, d, scale, causal, cu_seqlens};
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0) return -1;
    int64_t total = cu_seqlens ? (int64_t)Hq * N : (int64_t)B * Hq * N;
    if (!rows) nrows = total;
    int bad = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        int64_t cap = 0;
        double* s = NULL;
        double* qv = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 8)
        for (int64_t i = 0; i < nrows; ++i) {
            int64_t rowid = rows ? rows[i] : i;
            row_t r;
            if (rowid < 0 || rowid >= total || row_info(&a, rowid, &r) != 0) {
                bad = 1;
                continue;
            }
            if (r.len > cap) {
                free(s);
                cap = r.len;
                s = (double*)malloc(sizeof(double) * (size_t)cap);
            }
            for (int c = 0; c < d; ++c) qv[c] = bf16_to_double(r.qrow[c]);
            /* score row: s_j = scale * q . k_j, or -inf where masked */
            double m = -INFINITY;
            for (int64_t j = 0; j < r.len; ++j) {
                if (!key_allowed(&a, &r, j)) { s[j] = -INFINITY; continue; }
                const uint16_t* kj = r.k0 + j * r.kv_stride;
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += qv[c] * bf16_to_double(kj[c]);
                s[j] = scale * dot;
                if (s[j] > m) m = s[j];
            }
            double* orow = o + i * d;
            for (int c = 0; c < d; ++c) orow[c] = 0.0;
            if (m == -INFINITY) { lse[i] = -INFINITY; continue; }
            /* softmax of the row, then P V */
            double l = 0.0;
            for (int64_t j = 0; j < r.len; ++j) {
                s[j] = exp(s[j] - m);      /* exp(-inf) = 0 for masked keys */
                l += s[j];
            }
            for (int64_t j = 0; j < r.len; ++j) {
                if (s[j] == 0.0) continue;
                const uint16_t* vj = r.v0 + j * r.kv_stride;
                double pj = s[j] / l;
                for (int c = 0; c < d; ++c) orow[c] += pj * bf16_to_double(vj[c]);
            }
            lse[i] = m + log(l);
        }
        free(s);
        free(qv);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* The tiled forward of the 14cs17 page ("Flash Attention Algorithm"), in    */
/* fp64 and without any GPU concern: for each block of br query rows, start  */
/* with O = 0, l = 0, m = -inf; for each block of bc keys compute the score  */
/* block, fold it into (m, l, O) with the online-softmax update, and divide  */
/* O by l at the end.                                                        */
/*                                                                          */
/* The update equations (1)-(3) are missing from the extracted page; the    */
/* reading used here (m = max(m_old, m_blk), l = e^(m_old-m) l_old +         */
/* e^(m_blk-m) l_blk, O = e^(m_old-m) O_old + e^(m_blk-m) O_blk, with O kept */
/* unnormalised) is the rescale that Theorem 2's proof describes.            */
/*                                                                          */
/* kv_order: permutation of the key blocks (NULL: natural order); the       */
/* result must not depend on it.  Row ids and outputs as oracle_attention,  */
/* except that every row is computed (o is total_rows x d).                 */
/* ------------------------------------------------------------------------ */
int oracle_attention_tiled(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           int B, int Hq, int Hkv, int N, int d, double scale,
                           int causal, const int32_t* cu_seqlens,
                           int br, int bc, const int64_t* kv_order,
                           double* o, double* lse) {
    attn_t a = {q, k, v, B, Hq, Hkv, N, d, scale, causal, cu_seqlens};
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || br <= 0 || bc <= 0) return -1;
    int64_t total = cu_seqlens ? (int64_t)Hq * N : (int64_t)B * Hq * N;
    /* Walk the rows in query blocks of br consecutive row ids that share one
     * sequence and head. */
    double* Oacc = (double*)malloc(sizeof(double) * (size_t)br * d);
    double* mrow = (double*)malloc(sizeof(double) * (size_t)br);
    double* lrow = (double*)malloc(sizeof(double) * (size_t)br);
    double* sblk = (double*)malloc(sizeof(double) * (size_t)bc);
    int64_t rowid = 0;
    while (rowid < total) {
        row_t r0;
        if (row_info(&a, rowid, &r0) != 0) { rowid++; continue; }
        /* rows rowid .. rowid+nr-1 lie in the same sequence and head */
        int64_t nr = br;
        if (r0.t + nr > r0.len) nr = r0.len - r0.t;
        for (int64_t i = 0; i < nr; ++i) {
            mrow[i] = -INFINITY;
            lrow[i] = 0.0;
            for (int c = 0; c < d; ++c) Oacc[i * d + c] = 0.0;
        }
        int64_t nblk = (r0.len + bc - 1) / bc;
        for (int64_t tb = 0; tb < nblk; ++tb) {
            int64_t jb = kv_order ? kv_order[tb] : tb;
            if (jb >= nblk) continue;      /* permutation sized for a longer row */
            int64_t j0 = jb * bc, j1 = j0 + bc < r0.len ? j0 + bc : r0.len;
            for (int64_t i = 0; i < nr; ++i) {
                const uint16_t* qrow = r0.qrow + i * (a.cu ? (int64_t)Hq * d : d);
                /* S_ij for this query row and key block */
                double m_blk = -INFINITY;
                for (int64_t j = j0; j < j1; ++j) {
                    double sv = -INFINITY;
                    if (!causal || j <= r0.t + i) {
                        const uint16_t* kj = r0.k0 + j * r0.kv_stride;
                        double dot = 0.0;
                        for (int c = 0; c < d; ++c)
                            dot += bf16_to_double(qrow[c]) * bf16_to_double(kj[c]);
                        sv = scale * dot;
                    }
                    sblk[j - j0] = sv;
                    if (sv > m_blk) m_blk = sv;
                }
                if (m_blk == -INFINITY) continue;     /* block adds nothing */
                double m_new = mrow[i] > m_blk ? mrow[i] : m_blk;
                double c_old = (mrow[i] == -INFINITY) ? 0.0 : exp(mrow[i] - m_new);
                double c_blk = exp(m_blk - m_new);
                /* local block sums l_blk and O_blk, taken relative to m_blk */
                double l_blk = 0.0;
                double* Oi = Oacc + i * d;
                for (int c = 0; c < d; ++c) Oi[c] *= c_old;
                for (int64_t j = j0; j < j1; ++j) {
                    double pj = exp(sblk[j - j0] - m_blk);
                    if (pj == 0.0) continue;
                    l_blk += pj;
                    const uint16_t* vj = r0.v0 + j * r0.kv_stride;
                    for (int c = 0; c < d; ++c) Oi[c] += c_blk * pj * bf16_to_double(vj[c]);
                }
                lrow[i] = c_old * lrow[i] + c_blk * l_blk;
                mrow[i] = m_new;
            }
        }
        for (int64_t i = 0; i < nr; ++i) {
            double* orow = o + (rowid + i) * d;
            if (mrow[i] == -INFINITY) {
                for (int c = 0; c < d; ++c) orow[c] = 0.0;
                lse[rowid + i] = -INFINITY;
            } else {
                for (int c = 0; c < d; ++c) orow[c] = Oacc[i * d + c] / lrow[i];
                lse[rowid + i] = mrow[i] + log(lrow[i]);
            }
        }
        rowid += nr;
    }
    free(Oacc); free(mrow); free(lrow); free(sblk);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* A chunk of queries against a longer key sequence (xspy.com page, section  */
/* 1: chunked prefill splits a long prompt into chunks, each attending to    */
/* the keys of every earlier token; 14cs17 page: KV Cache is composable).    */
/* Query row i of the chunk sits at key position Nk - Nq + i; causal allows  */
/* key j iff j <= that position.  Dense layout: q [B,Hq,Nq,d],              */
/* k, v [B,Hkv,Nk,d]; row id (b*Hq + h)*Nq + i; o nrows x d, lse nrows.     */
/* Standard attention again: each score row is materialised in full.        */
/* ------------------------------------------------------------------------ */
int oracle_attention_kv(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        int B, int Hq, int Hkv, int Nq, int Nk, int d, double scale,
                        int causal, const int64_t* rows, int64_t nrows,
                        double* o, double* lse, int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || Nk < 0 || Nq < 0) return -1;
    const int group = Hq / Hkv;
    const int64_t total = (int64_t)B * Hq * Nq;
    if (!rows) nrows = total;
    int bad = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        double* qv = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 8)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t rowid = rows ? rows[r] : r;
            if (rowid < 0 || rowid >= total) { bad = 1; continue; }
            const int64_t i = rowid % Nq;
            const int64_t bh = rowid / Nq;
            const int h = (int)(bh % Hq);
            const int64_t b = bh / Hq;
            const int hk = h / group;
            const int64_t pos = (int64_t)Nk - Nq + i;          /* the row's key position */
            const uint16_t* qrow = q + ((b * Hq + h) * Nq + i) * d;
            const uint16_t* k0 = k + ((b * Hkv + hk) * (int64_t)Nk) * d;
            const uint16_t* v0 = v + ((b * Hkv + hk) * (int64_t)Nk) * d;
            for (int c = 0; c < d; ++c) qv[c] = bf16_to_double(qrow[c]);
            double m = -INFINITY;
            for (int64_t j = 0; j < Nk; ++j) {
                if (causal && j > pos) { s[j] = -INFINITY; continue; }
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += qv[c] * bf16_to_double(k0[j * d + c]);
                s[j] = scale * dot;
                if (s[j] > m) m = s[j];
            }
            double* orow = o + r * d;
            for (int c = 0; c < d; ++c) orow[c] = 0.0;
            if (m == -INFINITY) { lse[r] = -INFINITY; continue; }
            double l = 0.0;
            for (int64_t j = 0; j < Nk; ++j) {
                s[j] = exp(s[j] - m);
                l += s[j];
            }
            for (int64_t j = 0; j < Nk; ++j) {
                if (s[j] == 0.0) continue;
                double pj = s[j] / l;
                for (int c = 0; c < d; ++c) orow[c] += pj * bf16_to_double(v0[j * d + c]);
            }
            lse[r] = m + log(l);
        }
        free(s);
        free(qv);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* Gradients of standard attention (dense batches).                         */
/*                                                                          */
/* The pages say only that the backward pass recomputes the score matrix    */
/* from Q, K, V instead of storing it (14cs17 page, "Common Pitfalls",      */
/* Pitfall 3; fromzero2ai page, "Core Mechanisms of FlashAttention", item   */
/* 3).  What it computes is the derivative of the forward's definition:     */
/* with P = softmax(S) row-wise, S = scale Q K^T (masked entries -inf),     */
/* O = P V and an upstream gradient dO,                                     */
/*     dV = P^T dO,      dP = dO V^T,                                       */
/*     dS_ij = P_ij (dP_ij - D_i),  D_i = sum_j P_ij dP_ij                  */
/*             (the softmax Jacobian applied to row i of dP),               */
/*     dQ = scale dS K,  dK = scale dS^T Q.                                  */
/* Grouped-query attention: the Hq / Hkv query heads that read one          */
/* key/value head all add into that head's dK and dV.                        */
/*                                                                          */
/* Pass 1 walks the query rows: it materialises each score row, its         */
/* softmax, dP and dS in fp64 and forms dQ, keeping lse_i = m + log l and   */
/* D_i.  Pass 2 walks the keys: P_ij = exp(S_ij - lse_i) is the same        */
/* softmax entry, recomputed, and dK_j, dV_j sum over the query rows.       */
/*                                                                          */
/* units: list of nunits (batch, kv head) units b*Hkv + hk, or NULL for all */
/* (nunits is then B*Hkv).  Layouts: q, dout [B,Hq,N,d], k, v [B,Hkv,N,d].  */
/* Outputs per unit, in unit order: dq [group][N][d], dk and dv [N][d]      */
/* (with units == NULL that is dq [B,Hq,N,d], dk, dv [B,Hkv,N,d]).          */
/* A query row with no allowed key contributes nothing.  Returns 0, or -1   */
/* on bad arguments.                                                        */
/* ------------------------------------------------------------------------ */
int oracle_attention_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const uint16_t* dout, int B, int Hq, int Hkv, int N, int d,
                         double scale, int causal, const int64_t* units, int64_t nunits,
                         double* dq, double* dk, double* dv, int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || N < 0 || B < 0) return -1;
    const int group = Hq / Hkv;
    if (!units) nunits = (int64_t)B * Hkv;
    for (int64_t u = 0; u < nunits; ++u) {
        const int64_t unit = units ? units[u] : u;
        if (unit < 0 || unit >= (int64_t)B * Hkv) return -1;
    }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    const int64_t nd = (int64_t)N * d;
    double* Qw = (double*)malloc(sizeof(double) * (size_t)(group * nd + 1));
    double* Ow = (double*)malloc(sizeof(double) * (size_t)(group * nd + 1));   /* dO, widened */
    double* Kw = (double*)malloc(sizeof(double) * (size_t)(nd + 1));
    double* Vw = (double*)malloc(sizeof(double) * (size_t)(nd + 1));
    double* lse = (double*)malloc(sizeof(double) * (size_t)(group * (int64_t)N + 1));
    double* Dr = (double*)malloc(sizeof(double) * (size_t)(group * (int64_t)N + 1));
    if (!Qw || !Ow || !Kw || !Vw || !lse || !Dr) {
        free(Qw); free(Ow); free(Kw); free(Vw); free(lse); free(Dr);
        return -1;
    }
    for (int64_t u = 0; u < nunits; ++u) {
        const int64_t unit = units ? units[u] : u;
        const int64_t b = unit / Hkv;
        const int hk = (int)(unit % Hkv);
        const uint16_t* k0 = k + (b * Hkv + hk) * nd;
        const uint16_t* v0 = v + (b * Hkv + hk) * nd;
        for (int64_t e = 0; e < nd; ++e) {
            Kw[e] = bf16_to_double(k0[e]);
            Vw[e] = bf16_to_double(v0[e]);
        }
        for (int g = 0; g < group; ++g) {
            const int h = hk * group + g;
            const uint16_t* q0 = q + (b * Hq + h) * nd;
            const uint16_t* o0 = dout + (b * Hq + h) * nd;
            for (int64_t e = 0; e < nd; ++e) {
                Qw[g * nd + e] = bf16_to_double(q0[e]);
                Ow[g * nd + e] = bf16_to_double(o0[e]);
            }
        }
        double* dqu = dq + u * group * nd;
        double* dku = dk + u * nd;
        double* dvu = dv + u * nd;
        /* pass 1: query rows */
#pragma omp parallel
        {
            double* p = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
            double* dp = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#pragma omp for schedule(dynamic, 4)
            for (int64_t gi = 0; gi < (int64_t)group * N; ++gi) {
                const int64_t g = gi / N, i = gi % N;
                const double* qi = Qw + g * nd + i * d;
                const double* doi = Ow + g * nd + i * d;
                const int64_t nkeys = causal ? i + 1 : N;     /* keys j < nkeys allowed */
                double m = -INFINITY;
                for (int64_t j = 0; j < nkeys; ++j) {
                    double dot = 0.0;
                    for (int c = 0; c < d; ++c) dot += qi[c] * Kw[j * d + c];
                    p[j] = scale * dot;
                    if (p[j] > m) m = p[j];
                }
                double* dqi = dqu + g * nd + i * d;
                for (int c = 0; c < d; ++c) dqi[c] = 0.0;
                if (m == -INFINITY) { lse[gi] = -INFINITY; Dr[gi] = 0.0; continue; }
                double l = 0.0;
                for (int64_t j = 0; j < nkeys; ++j) {
                    p[j] = exp(p[j] - m);
                    l += p[j];
                }
                double D = 0.0;
                for (int64_t j = 0; j < nkeys; ++j) {
                    p[j] /= l;
                    double dot = 0.0;
                    for (int c = 0; c < d; ++c) dot += doi[c] * Vw[j * d + c];
                    dp[j] = dot;
                    D += p[j] * dp[j];
                }
                for (int64_t j = 0; j < nkeys; ++j) {
                    const double ds = p[j] * (dp[j] - D);
                    for (int c = 0; c < d; ++c) dqi[c] += scale * ds * Kw[j * d + c];
                }
                lse[gi] = m + log(l);
                Dr[gi] = D;
            }
            free(p);
            free(dp);
        }
        /* pass 2: keys */
#pragma omp parallel for schedule(dynamic, 4)
        for (int64_t j = 0; j < N; ++j) {
            double* dkj = dku + j * d;
            double* dvj = dvu + j * d;
            for (int c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
            const double* kj = Kw + j * d;
            const double* vj = Vw + j * d;
            for (int g = 0; g < group; ++g) {
                for (int64_t i = causal ? j : 0; i < N; ++i) {
                    const int64_t gi = (int64_t)g * N + i;
                    if (lse[gi] == -INFINITY) continue;
                    const double* qi = Qw + g * nd + i * d;
                    const double* doi = Ow + g * nd + i * d;
                    double s = 0.0, dp = 0.0;
                    for (int c = 0; c < d; ++c) {
                        s += qi[c] * kj[c];
                        dp += doi[c] * vj[c];
                    }
                    const double pij = exp(scale * s - lse[gi]);
                    const double ds = pij * (dp - Dr[gi]);
                    for (int c = 0; c < d; ++c) {
                        dvj[c] += pij * doi[c];
                        dkj[c] += scale * ds * qi[c];
                    }
                }
            }
        }
    }
    free(Qw); free(Ow); free(Kw); free(Vw); free(lse); free(Dr);
    return 0;
}

/* Number of worker threads OpenMP will use (reported by the CPU baseline). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
