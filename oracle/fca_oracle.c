/*
 * CPU oracle for Forest Cascade Attention (FCA) decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, calls or
 * includes this file; only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load it.  It shares no code, header or table
 * with the CUDA path.
 *
 * What it computes, and where that is defined:
 *
 *  - oracle_paged_attention: standard (non-cascaded) softmax attention of one
 *    decode query per (request, query head) over every cached token of that
 *    request, read through the request's block table.  FCA claims to be
 *    mathematically equivalent to exactly this ("ZoRRo Inference & Forest
 *    Cascade Attention", sections "Overview" and "Performance
 *    Characteristics"), so it is the reference for every attention output.
 *    The paged layout (fixed-size blocks, per-request block table that maps a
 *    logical block to a physical one) is the one of "PagedAttention vs.
 *    RadixAttention", section "How PagedAttention Works", steps 1-2.
 *    Readings where the pages are silent: scale is a caller argument (1/sqrt(D)
 *    by convention), the LSE is a natural log, query head h reads KV head
 *    h / (Hq/Hkv), no mask beyond the sequence length.
 *
 *  - oracle_attend / oracle_merge: attention over an explicit key set, and the
 *    weighted reduction of partial results by their log-sum-exp
 *    ("ZoRRo Inference & Forest Cascade Attention", "Core Mechanism" step 3;
 *    the same online-softmax merge is the correctness check of "Move the
 *    Query, Not the Cache", "Metodologia" item 4).
 *
 *  - oracle_plan: the group discovery step ("Core Mechanism" step 1) as a
 *    naive trie over each request's sequence of FULL physical block ids.  A
 *    trie node is a block-id prefix; its member set is the requests whose
 *    tables start with that prefix.  A group is a maximal run of trie depths
 *    over which the member set stays the same and has at least
 *    min_group_size members; nested groups form the forest.  Sharing means
 *    the same physical block id at the same logical index ("How PagedAttention
 *    Works" step 4: requests with the same prompt reference the same physical
 *    blocks; a block that will diverge is copied first, so only full blocks are
 *    shared).  Two options fold groups away (their interval passes to the
 *    groups below them, or to their members' own passes): min_shared_blocks
 *    (a group shorter than that) and min_saved_blocks (a group whose sharing
 *    saves fewer block reads, (members - 1) x length; the reading of FCA's
 *    automatic activation, "How It Works").
 *
 * All floating point is fp64 on the exact values of the bf16 inputs.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG -1
#define ORACLE_ERR_CAPACITY -2
#define ORACLE_ERR_NOMEM -3

/* bf16 bit pattern -> exact double */
static double bf16_bits_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------- */
/* Attention over an explicit key set                                         */
/* ------------------------------------------------------------------------- */

/*
 * o = sum_t softmax_t(s) * v_t with s_t = scale * <q, k_t>;
 * lse = log(sum_t exp(s_t)).  An empty key set gives lse = -inf and o = 0,
 * the identity element of the merge below.
 */
int oracle_attend(const double *q, const double *keys, const double *vals,
                  int64_t n, int32_t D, double scale, double *o, double *lse)
{
    if (D <= 0 || n < 0) return ORACLE_ERR_ARG;
    for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
    if (n == 0) {
        *lse = -INFINITY;
        return ORACLE_OK;
    }
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    if (!s) return ORACLE_ERR_NOMEM;
    double m = -INFINITY;
    for (int64_t t = 0; t < n; ++t) {
        double acc = 0.0;
        for (int32_t d = 0; d < D; ++d) acc += q[d] * keys[t * D + d];
        s[t] = scale * acc;
        if (s[t] > m) m = s[t];
    }
    double sum = 0.0;
    for (int64_t t = 0; t < n; ++t) sum += exp(s[t] - m);
    double l = m + log(sum);
    for (int64_t t = 0; t < n; ++t) {
        double p = exp(s[t] - l);
        for (int32_t d = 0; d < D; ++d) o[d] += p * vals[t * D + d];
    }
    *lse = l;
    free(s);
    return ORACLE_OK;
}

/*
 * Weighted reduction of partial results: lse = log(sum_i exp(lse_i)),
 * o = sum_i exp(lse_i - lse) * o_i.  Partials with lse_i = -inf (empty key
 * sets) carry no weight.
 */
int oracle_merge(const double *o_parts, const double *lse_parts, int32_t n_parts,
                 int32_t D, double *o, double *lse)
{
    if (D <= 0 || n_parts < 0) return ORACLE_ERR_ARG;
    for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
    double m = -INFINITY;
    for (int32_t i = 0; i < n_parts; ++i)
        if (lse_parts[i] > m) m = lse_parts[i];
    if (m == -INFINITY) {
        *lse = -INFINITY;
        return ORACLE_OK;
    }
    double sum = 0.0;
    for (int32_t i = 0; i < n_parts; ++i)
        if (lse_parts[i] != -INFINITY) sum += exp(lse_parts[i] - m);
    double l = m + log(sum);
    for (int32_t i = 0; i < n_parts; ++i) {
        if (lse_parts[i] == -INFINITY) continue;
        double w = exp(lse_parts[i] - l);
        for (int32_t d = 0; d < D; ++d) o[d] += w * o_parts[(int64_t)i * D + d];
    }
    *lse = l;
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Standard paged decode attention                                            */
/* ------------------------------------------------------------------------- */

/*
 * For each requested (r, h) pair (all R*Hq pairs, r-major, when pairs is
 * NULL): the keys and values are token positions t in [0, seq_lens[r]),
 * stored at cache[block_tables[r][t / B]][t % B][h / G][:], G = Hq / Hkv.
 * q is [R][Hq][D], caches are [num_blocks][B][Hkv][D], all bf16 bit patterns.
 * Outputs: out [n_pairs][D], lse [n_pairs], fp64.
 */
int oracle_paged_attention(const uint16_t *q, const uint16_t *k_cache,
                           const uint16_t *v_cache, const int32_t *block_tables,
                           int32_t max_blocks, const int32_t *seq_lens,
                           int32_t R, int32_t Hq, int32_t Hkv, int32_t D,
                           int32_t B, int64_t num_blocks, double scale,
                           const int32_t *pairs, int64_t n_pairs, double *out,
                           double *lse)
{
    if (R <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || B <= 0 || Hq % Hkv != 0)
        return ORACLE_ERR_ARG;
    if (!pairs) n_pairs = (int64_t)R * Hq;
    const int32_t G = Hq / Hkv;
    /* validate everything that will be read */
    for (int64_t i = 0; i < n_pairs; ++i) {
        int32_t r = pairs ? pairs[2 * i] : (int32_t)(i / Hq);
        int32_t h = pairs ? pairs[2 * i + 1] : (int32_t)(i % Hq);
        if (r < 0 || r >= R || h < 0 || h >= Hq) return ORACLE_ERR_ARG;
        int32_t L = seq_lens[r];
        if (L < 1 || (int64_t)L > (int64_t)max_blocks * B) return ORACLE_ERR_ARG;
        for (int32_t j = 0; j < (L + B - 1) / B; ++j) {
            int32_t blk = block_tables[(int64_t)r * max_blocks + j];
            if (blk < 0 || blk >= num_blocks) return ORACLE_ERR_ARG;
        }
    }
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n_pairs; ++i) {
        int32_t r = pairs ? pairs[2 * i] : (int32_t)(i / Hq);
        int32_t h = pairs ? pairs[2 * i + 1] : (int32_t)(i % Hq);
        int32_t kv = h / G;
        int32_t L = seq_lens[r];
        double *qd = (double *)malloc(sizeof(double) * (size_t)D);
        double *kd = (double *)malloc(sizeof(double) * (size_t)L * D);
        double *vd = (double *)malloc(sizeof(double) * (size_t)L * D);
        if (!qd || !kd || !vd) {
#pragma omp atomic write
            status = ORACLE_ERR_NOMEM;
            free(qd); free(kd); free(vd);
            continue;
        }
        for (int32_t d = 0; d < D; ++d)
            qd[d] = bf16_bits_to_double(q[((int64_t)r * Hq + h) * D + d]);
        for (int32_t t = 0; t < L; ++t) {
            int64_t blk = block_tables[(int64_t)r * max_blocks + t / B];
            int64_t base = ((blk * B + t % B) * Hkv + kv) * (int64_t)D;
            for (int32_t d = 0; d < D; ++d) {
                kd[(int64_t)t * D + d] = bf16_bits_to_double(k_cache[base + d]);
                vd[(int64_t)t * D + d] = bf16_bits_to_double(v_cache[base + d]);
            }
        }
        int rc = oracle_attend(qd, kd, vd, L, D, scale, out + i * D, lse + i);
        if (rc != ORACLE_OK) {
#pragma omp atomic write
            status = rc;
        }
        free(qd); free(kd); free(vd);
    }
    return status;
}

/* ------------------------------------------------------------------------- */
/* Group discovery: naive trie over full-block prefixes                      */
/* ------------------------------------------------------------------------- */

typedef struct {
    int32_t block;        /* physical block id on the edge into this node */
    int32_t depth;        /* number of blocks in the prefix (root = 0) */
    int32_t parent;
    int32_t first_child;
    int32_t next_sibling;
    int32_t count;        /* requests whose shareable prefix passes here */
} trie_node;

typedef struct {
    int32_t a, b;         /* block interval [a, b) the group reads */
    int32_t start_node;   /* trie node at depth (original chain start) */
    int32_t parent;       /* index into the emitted list, -1 for a root */
    int32_t min_member;
    int32_t n_members;
} raw_group;

typedef struct {
    trie_node *nodes;
    int32_t n_nodes, cap_nodes;
    raw_group *groups;
    int32_t n_groups, cap_groups;
    int32_t min_group_size, min_shared_blocks, min_saved_blocks;
} trie_state;

static int32_t trie_child(trie_state *st, int32_t v, int32_t block)
{
    for (int32_t c = st->nodes[v].first_child; c >= 0; c = st->nodes[c].next_sibling)
        if (st->nodes[c].block == block) return c;
    if (st->n_nodes == st->cap_nodes) return -1;
    int32_t c = st->n_nodes++;
    st->nodes[c].block = block;
    st->nodes[c].depth = st->nodes[v].depth + 1;
    st->nodes[c].parent = v;
    st->nodes[c].first_child = -1;
    st->nodes[c].count = 0;
    st->nodes[c].next_sibling = st->nodes[v].first_child;
    st->nodes[v].first_child = c;
    return c;
}

/* the child of v that keeps all of v's members, or -1 */
static int32_t same_set_child(const trie_state *st, int32_t v)
{
    for (int32_t c = st->nodes[v].first_child; c >= 0; c = st->nodes[c].next_sibling)
        if (st->nodes[c].count == st->nodes[v].count) return c;
    return -1;
}

/*
 * Depth-first walk over chains.  A chain starts at a node whose member set
 * differs from its parent's (or at depth 1) and follows the unique child with
 * the same member set down to its last node.  Chains with fewer than
 * min_group_size members are not groups, and neither is anything below them.
 * A chain shorter than min_shared_blocks (after absorbing any dropped
 * ancestors, "pending"), or one whose sharing saves fewer than
 * min_saved_blocks block reads ((members - 1) x its length in blocks: the
 * reads of the shared blocks by all but one member), is dropped: its interval
 * passes to the chains below it, or stays with the members' suffixes if there
 * are none.
 */
static int walk_chain(trie_state *st, int32_t start, int32_t parent_group, int32_t pending)
{
    trie_node *nd = st->nodes;
    if (nd[start].count < st->min_group_size) return ORACLE_OK;
    int32_t a = nd[start].depth - 1;
    int32_t end = start;
    for (int32_t c = same_set_child(st, end); c >= 0; c = same_set_child(st, end)) end = c;
    int32_t b = nd[end].depth;
    int32_t eff_a = pending >= 0 ? pending : a;
    int32_t next_parent = parent_group, next_pending = -1;
    if (b - eff_a < st->min_shared_blocks ||
        (int64_t)(nd[start].count - 1) * (b - eff_a) < (int64_t)st->min_saved_blocks) {
        next_pending = eff_a;
    } else {
        if (st->n_groups == st->cap_groups) return ORACLE_ERR_CAPACITY;
        raw_group *g = &st->groups[st->n_groups];
        g->a = eff_a;
        g->b = b;
        g->start_node = start;
        g->parent = parent_group;
        g->n_members = nd[start].count;
        g->min_member = -1;
        next_parent = st->n_groups++;
    }
    for (int32_t c = nd[end].first_child; c >= 0; c = nd[c].next_sibling) {
        int rc = walk_chain(st, c, next_parent, next_pending);
        if (rc != ORACLE_OK) return rc;
    }
    return ORACLE_OK;
}

static const raw_group *g_sort_base;
static int cmp_group_idx(const void *x, const void *y)
{
    const raw_group *gx = &g_sort_base[*(const int32_t *)x];
    const raw_group *gy = &g_sort_base[*(const int32_t *)y];
    if (gx->a != gy->a) return gx->a < gy->a ? -1 : 1;
    if (gx->min_member != gy->min_member) return gx->min_member < gy->min_member ? -1 : 1;
    return 0;
}

/*
 * Inputs: block_tables [R][max_blocks] int32, seq_lens [R] (1 <= L <= max_blocks*B).
 * Request r's shareable sequence is block_tables[r][0 : seq_lens[r] / B]
 * (full blocks only).
 * Outputs, in canonical order (groups by (a ascending, smallest member
 * ascending); members of each group ascending; parent as an index in that
 * order, -1 for roots):
 *   *n_groups, g_a[], g_b[], g_parent[], g_member_off[], g_n_members[]
 *   members[] (concatenated), suffix_start[R] (in blocks; the b of the
 *   deepest group containing r, else 0).
 * Capacities: cap_groups entries for the g_* arrays, cap_members for
 * members[].  Returns 0, or a negative code.
 */
int oracle_plan(const int32_t *block_tables, int32_t R, int32_t max_blocks,
                const int32_t *seq_lens, int32_t B, int32_t min_group_size,
                int32_t min_shared_blocks, int32_t min_saved_blocks, int32_t *n_groups, int32_t *g_a,
                int32_t *g_b, int32_t *g_parent, int32_t *g_member_off,
                int32_t *g_n_members, int32_t *members, int32_t *suffix_start,
                int32_t cap_groups, int64_t cap_members)
{
    if (R <= 0 || max_blocks <= 0 || B <= 0 || min_group_size < 2 || min_shared_blocks < 1 ||
        min_saved_blocks < 0)
        return ORACLE_ERR_ARG;
    int64_t total_full = 0;
    for (int32_t r = 0; r < R; ++r) {
        if (seq_lens[r] < 1 || (int64_t)seq_lens[r] > (int64_t)max_blocks * B) return ORACLE_ERR_ARG;
        total_full += seq_lens[r] / B;
    }
    trie_state st;
    memset(&st, 0, sizeof st);
    st.cap_nodes = (int32_t)(total_full + 1);
    st.nodes = (trie_node *)malloc(sizeof(trie_node) * (size_t)st.cap_nodes);
    st.cap_groups = R;  /* a laminar family of sets of size >= 2 over R items has < R sets */
    st.groups = (raw_group *)malloc(sizeof(raw_group) * (size_t)st.cap_groups);
    int32_t *path_node = (int32_t *)malloc(sizeof(int32_t) * (size_t)(total_full + 1));
    int64_t *path_off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(R + 1));
    if (!st.nodes || !st.groups || !path_node || !path_off) {
        free(st.nodes); free(st.groups); free(path_node); free(path_off);
        return ORACLE_ERR_NOMEM;
    }
    st.min_group_size = min_group_size;
    st.min_shared_blocks = min_shared_blocks;
    st.min_saved_blocks = min_saved_blocks;
    st.n_nodes = 1;
    st.nodes[0].block = -1;
    st.nodes[0].depth = 0;
    st.nodes[0].parent = -1;
    st.nodes[0].first_child = -1;
    st.nodes[0].next_sibling = -1;
    st.nodes[0].count = R;

    /* insert every request's full-block sequence */
    path_off[0] = 0;
    for (int32_t r = 0; r < R; ++r) {
        int32_t n_full = seq_lens[r] / B;
        int32_t v = 0;
        for (int32_t j = 0; j < n_full; ++j) {
            v = trie_child(&st, v, block_tables[(int64_t)r * max_blocks + j]);
            st.nodes[v].count += 1;
            path_node[path_off[r] + j] = v;
        }
        path_off[r + 1] = path_off[r] + n_full;
    }

    int rc = ORACLE_OK;
    for (int32_t c = st.nodes[0].first_child; c >= 0 && rc == ORACLE_OK; c = st.nodes[c].next_sibling)
        rc = walk_chain(&st, c, -1, -1);
    if (rc != ORACLE_OK) goto done;
    if (st.n_groups > cap_groups) { rc = ORACLE_ERR_CAPACITY; goto done; }

    /* members of a group = requests whose path passes the chain's start node */
    int64_t total_members = 0;
    for (int32_t g = 0; g < st.n_groups; ++g) total_members += st.groups[g].n_members;
    if (total_members > cap_members) { rc = ORACLE_ERR_CAPACITY; goto done; }
    for (int32_t g = 0; g < st.n_groups; ++g) {
        int32_t v = st.groups[g].start_node, dv = st.nodes[v].depth;
        for (int32_t r = 0; r < R; ++r)
            if (path_off[r + 1] - path_off[r] >= dv && path_node[path_off[r] + dv - 1] == v) {
                st.groups[g].min_member = r;
                break;
            }
    }

    /* canonical order */
    int32_t *order = (int32_t *)malloc(sizeof(int32_t) * (size_t)(st.n_groups + 1));
    int32_t *rank = (int32_t *)malloc(sizeof(int32_t) * (size_t)(st.n_groups + 1));
    if (!order || !rank) { free(order); free(rank); rc = ORACLE_ERR_NOMEM; goto done; }
    for (int32_t g = 0; g < st.n_groups; ++g) order[g] = g;
    g_sort_base = st.groups;
    qsort(order, (size_t)st.n_groups, sizeof(int32_t), cmp_group_idx);
    for (int32_t i = 0; i < st.n_groups; ++i) rank[order[i]] = i;

    for (int32_t r = 0; r < R; ++r) suffix_start[r] = 0;
    int64_t off = 0;
    for (int32_t i = 0; i < st.n_groups; ++i) {
        const raw_group *g = &st.groups[order[i]];
        g_a[i] = g->a;
        g_b[i] = g->b;
        g_parent[i] = g->parent < 0 ? -1 : rank[g->parent];
        g_member_off[i] = (int32_t)off;
        g_n_members[i] = g->n_members;
        int32_t v = g->start_node, dv = st.nodes[v].depth;
        for (int32_t r = 0; r < R; ++r) {
            if (path_off[r + 1] - path_off[r] >= dv && path_node[path_off[r] + dv - 1] == v) {
                members[off++] = r;
                if (g->b > suffix_start[r]) suffix_start[r] = g->b;
            }
        }
    }
    *n_groups = st.n_groups;
    free(order);
    free(rank);
done:
    free(st.nodes);
    free(st.groups);
    free(path_node);
    free(path_off);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* Byte accounting                                                            */
/* ------------------------------------------------------------------------- */

/*
 * Unique KV tokens of a batch: every distinct physical block referenced by
 * the first ceil(L_r / B) entries of some table, counted once, with the
 * largest number of valid tokens any referencing request has in it.
 * Multiply by Hkv * D * 2 (K and V) * 2 bytes for unique KV bytes.
 */
int64_t oracle_unique_kv_tokens(const int32_t *block_tables, int32_t R, int32_t max_blocks,
                                const int32_t *seq_lens, int32_t B, int64_t num_blocks)
{
    if (R <= 0 || B <= 0 || num_blocks <= 0) return ORACLE_ERR_ARG;
    int32_t *valid = (int32_t *)calloc((size_t)num_blocks, sizeof(int32_t));
    if (!valid) return ORACLE_ERR_NOMEM;
    for (int32_t r = 0; r < R; ++r) {
        int32_t L = seq_lens[r];
        if (L < 1 || (int64_t)L > (int64_t)max_blocks * B) { free(valid); return ORACLE_ERR_ARG; }
        for (int32_t j = 0; j < (L + B - 1) / B; ++j) {
            int32_t blk = block_tables[(int64_t)r * max_blocks + j];
            if (blk < 0 || blk >= num_blocks) { free(valid); return ORACLE_ERR_ARG; }
            int32_t n = L - j * B < B ? L - j * B : B;
            if (n > valid[blk]) valid[blk] = n;
        }
    }
    int64_t total = 0;
    for (int64_t b = 0; b < num_blocks; ++b) total += valid[b];
    free(valid);
    return total;
}

/* Threads of the OpenMP loop in oracle_paged_attention (timing only; the
 * result does not depend on it).  Returns the count in force before. */
int oracle_set_threads(int n)
{
#ifdef _OPENMP
    int before = omp_get_max_threads();
    if (n > 0)
        omp_set_num_threads(n);
    return before;
#else
    (void)n;
    return 1;
#endif
}
