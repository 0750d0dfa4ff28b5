/*
 * Oracle (test infrastructure only; never linked into the product library).
 *
 * Plain fp64 tree attention written from its definition.  JetSpec README,
 * "JetSpec / Overview": the target verifies the whole draft tree in one
 * forward pass under a tree-causal attention mask.  Read plainly, node i of a
 * request sees exactly what a causal decoder would see if the sequence were
 * the committed prefix followed by the root-to-i path of the tree:
 *
 *   S(i)   = [prefix slots 0..P-1] ++ [slot P + j for j on root..i]
 *   s_j    = scale * <q_{i,h}, k_{j,g}>,  g = h / (Hq / Hkv)
 *   o_{i,h} = sum_j softmax(s)_j v_{j,g}
 *
 * Tree node j's key/value live at logical cache slot P + j; logical slot s of
 * request b lives in physical page page_table[b][s / 16], row s % 16, of a
 * cache laid out [num_pages][16][Hkv][D].
 *
 * Every row is computed on its own, in the order written above, in double
 * precision; bf16 inputs convert exactly.  Threads only split the list of
 * rows.  No blocking, fusion or reordering.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

typedef struct {
    int B, Hq, Hkv, D, page_size, max_pages_per_req;
    const int32_t *page_table, *prefix_len, *node_offsets, *parent;
    const uint16_t *q, *k_cache, *v_cache;
    double scale;
    const int32_t *rows;   /* [nrows][2] = (global node t, query head h) */
    int nrows;
    double *out;           /* [nrows][D] */
    int next;              /* work counter */
    pthread_mutex_t lock;
    int status;            /* 0 ok, nonzero = malformed input seen */
} job_t;

/* Address of element 0 of (request b, logical slot s, kv head g). */
static const uint16_t *slot_row(const job_t *a, const uint16_t *cache, int b, int s, int g)
{
    int page = a->page_table[(size_t)b * a->max_pages_per_req + s / a->page_size];
    size_t phys = (size_t)page * a->page_size + (size_t)(s % a->page_size);
    return cache + (phys * a->Hkv + g) * a->D;
}

static int request_of(const job_t *a, int t)
{
    for (int b = 0; b < a->B; ++b)
        if (t >= a->node_offsets[b] && t < a->node_offsets[b + 1]) return b;
    return -1;
}

static int one_row(const job_t *a, int t, int h, double *o)
{
    int b = request_of(a, t);
    if (b < 0) return 1;
    int base = a->node_offsets[b];
    int n = a->node_offsets[b + 1] - base;
    int P = a->prefix_len[b];
    int i = t - base;
    int g = h / (a->Hq / a->Hkv);
    int D = a->D;

    /* root..i path, as request-local node indices */
    int *path = (int *)malloc(sizeof(int) * (size_t)(n + 1));
    int len = 0;
    for (int j = i; j != -1; j = a->parent[base + j]) {
        if (len > n) { free(path); return 1; }
        path[len++] = j;
    }
    for (int x = 0; x < len / 2; ++x) {
        int tmp = path[x];
        path[x] = path[len - 1 - x];
        path[len - 1 - x] = tmp;
    }

    int L = P + len;
    double *s = (double *)malloc(sizeof(double) * (size_t)L);
    const uint16_t *qv = a->q + ((size_t)t * a->Hq + h) * D;
    for (int j = 0; j < L; ++j) {
        int slot = j < P ? j : P + path[j - P];
        const uint16_t *kr = slot_row(a, a->k_cache, b, slot, g);
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += bf16_to_f64(qv[d]) * bf16_to_f64(kr[d]);
        s[j] = a->scale * dot;
    }
    double m = -INFINITY;
    for (int j = 0; j < L; ++j) m = s[j] > m ? s[j] : m;
    double denom = 0.0;
    for (int j = 0; j < L; ++j) {
        s[j] = exp(s[j] - m);
        denom += s[j];
    }
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int j = 0; j < L; ++j) {
        int slot = j < P ? j : P + path[j - P];
        const uint16_t *vr = slot_row(a, a->v_cache, b, slot, g);
        for (int d = 0; d < D; ++d) o[d] += s[j] * bf16_to_f64(vr[d]);
    }
    for (int d = 0; d < D; ++d) o[d] /= denom;
    free(s);
    free(path);
    return 0;
}

static void *worker(void *arg)
{
    job_t *a = (job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&a->lock);
        int r = a->next++;
        pthread_mutex_unlock(&a->lock);
        if (r >= a->nrows) break;
        int bad = one_row(a, a->rows[2 * r], a->rows[2 * r + 1], a->out + (size_t)r * a->D);
        if (bad) {
            pthread_mutex_lock(&a->lock);
            a->status = 1;
            pthread_mutex_unlock(&a->lock);
        }
    }
    return NULL;
}

/* Returns 0 on success, 1 if a row's request or path was malformed. */
int oracle_tree_attention(int B, int Hq, int Hkv, int D, int page_size, int max_pages_per_req,
                          const int32_t *page_table, const int32_t *prefix_len,
                          const int32_t *node_offsets, const int32_t *parent,
                          const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                          double scale, const int32_t *rows, int nrows, double *out,
                          int nthreads)
{
    job_t a;
    memset(&a, 0, sizeof a);
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.page_size = page_size;
    a.max_pages_per_req = max_pages_per_req;
    a.page_table = page_table; a.prefix_len = prefix_len; a.node_offsets = node_offsets;
    a.parent = parent; a.q = q; a.k_cache = k_cache; a.v_cache = v_cache; a.scale = scale;
    a.rows = rows; a.nrows = nrows; a.out = out;
    pthread_mutex_init(&a.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &a);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&a.lock);
    return a.status;
}
