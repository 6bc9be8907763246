/*
 * dms_oracle.c - plain, slow CPU oracle for the DMS decode path (fp64).
 *
 * TEST INFRASTRUCTURE: see dms_oracle.h. Nothing here is tuned; loops are
 * written to be checked by eye against the definitions they state.
 */
#include "dms_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Delayed eviction ("Inference-Time Hyper-Scaling with KV Cache
 * Compression", paper summary, Key claims and Method, section 3.2): the
 * decision alpha_j taken for token j acts only after w further steps.
 * A kept token (alpha_j == 0) stays forever. */
int dmso_visible(long s, long j, int alpha_j, int window) {
    if (j < 0 || j > s) return 0;
    if (alpha_j == 0) return 1;
    return (s - j) < window;
}

/* Eviction as an additive mask on attention logits (paper summary, Method;
 * section 3.2 "Performance Considerations"): -inf where not visible, then an
 * ordinary softmax over positions and a weighted sum of value rows. */
void dmso_attention(int T, int window, int d, int g, const double* q,
                    const double* K, const double* V, const unsigned char* alpha,
                    double scale, double* out) {
    long s = (long)T - 1;
    double* logit = (double*)malloc(sizeof(double) * (T > 0 ? (size_t)T : 1));
    for (int h = 0; h < g; ++h) {
        const double* qh = q + (size_t)h * d;
        double* oh = out + (size_t)h * d;
        for (int c = 0; c < d; ++c) oh[c] = 0.0;

        double mx = -INFINITY;
        int any = 0;
        for (long j = 0; j <= s; ++j) {
            if (!dmso_visible(s, j, alpha[j] != 0, window)) {
                logit[j] = -INFINITY;
                continue;
            }
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += qh[c] * K[(size_t)j * d + c];
            logit[j] = scale * dot;
            if (logit[j] > mx) mx = logit[j];
            any = 1;
        }
        if (!any) continue;

        double den = 0.0;
        for (long j = 0; j <= s; ++j) {
            if (logit[j] == -INFINITY) continue;
            double e = exp(logit[j] - mx);
            den += e;
            for (int c = 0; c < d; ++c) oh[c] += e * V[(size_t)j * d + c];
        }
        for (int c = 0; c < d; ++c) oh[c] /= den;
    }
    free(logit);
}

int dmso_attention_batch(int n, const int* T, int window, int d, int g,
                         const double* const* q, const double* const* K,
                         const double* const* V, const unsigned char* const* alpha,
                         double scale, double* const* out) {
    int threads = 1;
#ifdef _OPENMP
#pragma omp parallel
    {
#pragma omp single
        threads = omp_get_num_threads();
    }
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int i = 0; i < n; ++i) {
        dmso_attention(T[i], window, d, g, q[i], K[i], V[i], alpha[i], scale, out[i]);
    }
    return threads;
}

/* ------------------------------------------------------------------------ */
/* Slot-pool simulator. Every stream remembers, for every position it has
 * ever seen, the logical slot and the decision of that token, so the token
 * that leaves at step s is found by direct lookup of position s - w. */

typedef struct {
    int pos;            /* tokens seen */
    int n;              /* logical slots in use = retained tokens */
    int n_pages;
    int cap;            /* allocated length of tok_slot / tok_alpha */
    int* tok_slot;      /* logical slot of each position */
    unsigned char* tok_alpha;
} dmso_stream;

struct dmso_sim {
    int max_seqs, hkv, w, P, max_pages, mps;
    dmso_stream* st;    /* [max_seqs * hkv] */
    int* page_table;    /* [S][mps] */
    int* slot_pos;      /* [max_pages * P] */
    int* free_list;     /* stack, top at free_count - 1 */
    int free_count;
};

dmso_sim* dmso_sim_create(int max_seqs, int num_kv_heads, int window, int page_size,
                          int max_pages, int max_pages_per_stream) {
    if (max_seqs <= 0 || num_kv_heads <= 0 || window <= 0 || page_size <= 0 ||
        max_pages <= 0 || max_pages_per_stream <= 0)
        return NULL;
    dmso_sim* sim = (dmso_sim*)calloc(1, sizeof(dmso_sim));
    int S = max_seqs * num_kv_heads;
    sim->max_seqs = max_seqs;
    sim->hkv = num_kv_heads;
    sim->w = window;
    sim->P = page_size;
    sim->max_pages = max_pages;
    sim->mps = max_pages_per_stream;
    sim->st = (dmso_stream*)calloc((size_t)S, sizeof(dmso_stream));
    sim->page_table = (int*)malloc(sizeof(int) * (size_t)S * max_pages_per_stream);
    for (size_t i = 0; i < (size_t)S * max_pages_per_stream; ++i) sim->page_table[i] = -1;
    sim->slot_pos = (int*)malloc(sizeof(int) * (size_t)max_pages * page_size);
    for (size_t i = 0; i < (size_t)max_pages * page_size; ++i) sim->slot_pos[i] = -1;
    /* A fresh stack pops 0, 1, 2, ...: page k sits k places below the top. */
    sim->free_list = (int*)malloc(sizeof(int) * (size_t)max_pages);
    for (int i = 0; i < max_pages; ++i) sim->free_list[i] = max_pages - 1 - i;
    sim->free_count = max_pages;
    return sim;
}

void dmso_sim_destroy(dmso_sim* sim) {
    if (!sim) return;
    int S = sim->max_seqs * sim->hkv;
    for (int i = 0; i < S; ++i) {
        free(sim->st[i].tok_slot);
        free(sim->st[i].tok_alpha);
    }
    free(sim->st);
    free(sim->page_table);
    free(sim->slot_pos);
    free(sim->free_list);
    free(sim);
}

static void grow(dmso_stream* t, int need) {
    if (need <= t->cap) return;
    int cap = t->cap ? t->cap : 64;
    while (cap < need) cap *= 2;
    t->tok_slot = (int*)realloc(t->tok_slot, sizeof(int) * (size_t)cap);
    t->tok_alpha = (unsigned char*)realloc(t->tok_alpha, (size_t)cap);
    t->cap = cap;
}

/* Append one token with decision a to stream id. Returns status; on success
 * *phys receives the physical slot written. */
static int append_one(dmso_sim* sim, int id, int a, int* phys) {
    dmso_stream* t = &sim->st[id];
    int s = t->pos;
    int slot;
    if (s >= sim->w && t->tok_alpha[s - sim->w] == 1) {
        /* token s - w leaves the cache now; s reuses its slot */
        slot = t->tok_slot[s - sim->w];
    } else {
        slot = t->n;
        if (slot % sim->P == 0) {
            int page_index = slot / sim->P;
            if (page_index >= sim->mps) return DMSO_ERR_STREAM_FULL;
            if (sim->free_count == 0) return DMSO_ERR_POOL_EXHAUSTED;
            sim->free_count -= 1;
            sim->page_table[(size_t)id * sim->mps + page_index] = sim->free_list[sim->free_count];
            t->n_pages += 1;
        }
        t->n += 1;
    }
    grow(t, s + 1);
    t->tok_slot[s] = slot;
    t->tok_alpha[s] = (unsigned char)(a != 0);
    t->pos = s + 1;
    int p = sim->page_table[(size_t)id * sim->mps + slot / sim->P] * sim->P + slot % sim->P;
    sim->slot_pos[p] = s;
    if (phys) *phys = p;
    return DMSO_OK;
}

int dmso_sim_append(dmso_sim* sim, int n_seqs, const int* seq_ids, const int* counts,
                    const unsigned char* alpha, int* phys_slot) {
    long base = 0;  /* first token of seq i in the call */
    for (int i = 0; i < n_seqs; ++i) {
        if (seq_ids[i] < 0 || seq_ids[i] >= sim->max_seqs || counts[i] < 0) return DMSO_ERR_INVALID;
        for (int h = 0; h < sim->hkv; ++h) {
            int id = seq_ids[i] * sim->hkv + h;
            for (int k = 0; k < counts[i]; ++k) {
                size_t at = (size_t)(base + k) * sim->hkv + h;
                int phys = -1;
                int rc = append_one(sim, id, alpha[at], &phys);
                if (rc != DMSO_OK) return rc;
                if (phys_slot) phys_slot[at] = phys;
            }
        }
        base += counts[i];
    }
    return DMSO_OK;
}

int dmso_sim_reset_seq(dmso_sim* sim, int seq_id) {
    if (seq_id < 0 || seq_id >= sim->max_seqs) return DMSO_ERR_INVALID;
    for (int h = 0; h < sim->hkv; ++h) {
        int id = seq_id * sim->hkv + h;
        dmso_stream* t = &sim->st[id];
        for (int p = t->n_pages - 1; p >= 0; --p) {
            int* e = &sim->page_table[(size_t)id * sim->mps + p];
            sim->free_list[sim->free_count++] = *e;
            *e = -1;
        }
        t->pos = 0;
        t->n = 0;
        t->n_pages = 0;
    }
    return DMSO_OK;
}

void dmso_sim_snapshot(const dmso_sim* sim, int* page_table, int* n_pages, int* n, int* pos,
                       int* slot_pos, int* free_list, int* free_count) {
    int S = sim->max_seqs * sim->hkv;
    if (page_table) memcpy(page_table, sim->page_table, sizeof(int) * (size_t)S * sim->mps);
    for (int i = 0; i < S; ++i) {
        if (n_pages) n_pages[i] = sim->st[i].n_pages;
        if (n) n[i] = sim->st[i].n;
        if (pos) pos[i] = sim->st[i].pos;
    }
    if (slot_pos) memcpy(slot_pos, sim->slot_pos, sizeof(int) * (size_t)sim->max_pages * sim->P);
    if (free_list) memcpy(free_list, sim->free_list, sizeof(int) * (size_t)sim->max_pages);
    if (free_count) *free_count = sim->free_count;
}

int dmso_sim_retained(const dmso_sim* sim, int stream, int* positions) {
    const dmso_stream* t = &sim->st[stream];
    for (int l = 0; l < t->n; ++l) {
        int p = sim->page_table[(size_t)stream * sim->mps + l / sim->P] * sim->P + l % sim->P;
        positions[l] = sim->slot_pos[p];
    }
    return t->n;
}
