/*
 * Oracle (test infrastructure only): plain fp64 CPU definitions of the
 * Geo-FlashAttention patch pipeline.  Only tests/, the smoke check and the
 * bench's CPU baseline may load this.  It shares no code with the CUDA path.
 *
 * Source: "Spatial-Spectral Coupling as Attention" project page, section
 * "Geo-FlashAttention" (pipeline: partition both shapes into geodesic patches,
 * pool source keys, score source patches, keep the top R per target patch) and
 * the ai4snews digest, "Interpretation" (geodesic farthest-point sampling).
 *
 * Readings taken where the pages are silent:
 *  - geodesic distance on the synthetic sphere is the great-circle distance,
 *    which decreases monotonically with the dot product, so every ranking is
 *    done on the fp64 dot ((x0*y0 + x1*y1) + x2*y2) of the fp32 coordinates
 *    (each product of two fp32 values is exact in fp64);
 *  - FPS starts at the given seed vertex; each next centre is the vertex not
 *    yet chosen whose largest dot to the chosen centres is smallest (farthest
 *    point), ties to the lowest vertex index;
 *  - the patch of a vertex is its nearest centre (largest dot), ties to the
 *    lowest patch index; a centre always belongs to its own patch;
 *  - pooling is the mean: fp64 sum in ascending vertex order, one division;
 *  - score(p,q) = <mean_N(p), mean_M(q)>, summed over c = 0..d-1 in order;
 *  - top R: the R largest scores of a row, ties to the lower source patch,
 *    listed by (score descending, patch ascending).
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared (see oracle/build.py).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

static double dot3(const float* a, const float* b) {
    double p0 = (double)a[0] * (double)b[0];
    double p1 = (double)a[1] * (double)b[1];
    double p2 = (double)a[2] * (double)b[2];
    return (p0 + p1) + p2;
}

/* Farthest-point sampling plus nearest-centre assignment.
 * pts [n,3] fp32; centers [P]; owner [n]; maxdot [n] (nullable) receives the
 * final largest dot of every vertex to the centres.  Returns 0, or -1 on bad
 * arguments. */
int oracle_fps(const float* pts, int n, int P, int seed, int* centers, int* owner,
               double* maxdot_out) {
    if (n < 1 || P < 1 || P > n || seed < 0 || seed >= n) return -1;
    double* best = (double*)malloc(sizeof(double) * (size_t)n);
    unsigned char* chosen = (unsigned char*)calloc((size_t)n, 1);
    if (!best || !chosen) { free(best); free(chosen); return -1; }
    for (int v = 0; v < n; ++v) { best[v] = -INFINITY; owner[v] = -1; }
    int c = seed;
    for (int t = 0; t < P; ++t) {
        centers[t] = c;
        chosen[c] = 1;
        owner[c] = t;
        const float* xc = pts + 3 * (size_t)c;
        for (int v = 0; v < n; ++v) {
            if (chosen[v]) continue;
            double g = dot3(pts + 3 * (size_t)v, xc);
            if (g > best[v]) { best[v] = g; owner[v] = t; }
        }
        if (t + 1 == P) break;
        int arg = -1;
        double lo = INFINITY;
        for (int v = 0; v < n; ++v) {
            if (chosen[v]) continue;
            if (arg < 0 || best[v] < lo) { lo = best[v]; arg = v; }
        }
        c = arg;
    }
    if (maxdot_out) {
        for (int v = 0; v < n; ++v)
            maxdot_out[v] = chosen[v] ? dot3(pts + 3 * (size_t)v, pts + 3 * (size_t)v) : best[v];
    }
    free(best);
    free(chosen);
    return 0;
}

/* Patch lists: offsets [P+1] (prefix sums of patch sizes), members [n] holding
 * the vertices of patch 0, then patch 1, ..., each in ascending vertex order. */
int oracle_csr(const int* owner, int n, int P, int* offsets, int* members) {
    for (int p = 0; p <= P; ++p) offsets[p] = 0;
    for (int v = 0; v < n; ++v) {
        if (owner[v] < 0 || owner[v] >= P) return -1;
        offsets[owner[v] + 1] += 1;
    }
    for (int p = 0; p < P; ++p) offsets[p + 1] += offsets[p];
    int* fill = (int*)malloc(sizeof(int) * (size_t)P);
    if (!fill) return -1;
    for (int p = 0; p < P; ++p) fill[p] = offsets[p];
    for (int v = 0; v < n; ++v) members[fill[owner[v]]++] = v;
    free(fill);
    return 0;
}

/* Mean descriptor of every patch: F [n,d] (already widened to fp64), mu [P,d]. */
int oracle_pool(const double* F, int n, int d, const int* offsets, const int* members,
                int P, double* mu) {
    for (int p = 0; p < P; ++p) {
        int b = offsets[p], e = offsets[p + 1];
        if (e <= b) return -1;
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            for (int r = b; r < e; ++r) {
                int v = members[r];
                if (v < 0 || v >= n) return -1;
                s = s + F[(size_t)v * d + c];
            }
            mu[(size_t)p * d + c] = s / (double)(e - b);
        }
    }
    return 0;
}

/* scores [PN,PM]: dot of the mean descriptors, summed over c in order. */
void oracle_scores(const double* muN, int PN, const double* muM, int PM, int d,
                   double* scores) {
    for (int p = 0; p < PN; ++p)
        for (int q = 0; q < PM; ++q) {
            double s = 0.0;
            for (int c = 0; c < d; ++c) {
                double t = muN[(size_t)p * d + c] * muM[(size_t)q * d + c];
                s = s + t;
            }
            scores[(size_t)p * PM + q] = s;
        }
}

static const double* g_row;
static int cmp_desc(const void* a, const void* b) {
    int qa = *(const int*)a, qb = *(const int*)b;
    double sa = g_row[qa], sb = g_row[qb];
    if (sa > sb) return -1;
    if (sa < sb) return 1;
    return (qa < qb) ? -1 : (qa > qb);
}

/* topk [PN,R]: per row the R best source patches, (score desc, index asc). */
int oracle_topk(const double* scores, int PN, int PM, int R, int* topk) {
    if (R < 1 || R > PM) return -1;
    int* idx = (int*)malloc(sizeof(int) * (size_t)PM);
    if (!idx) return -1;
    for (int p = 0; p < PN; ++p) {
        for (int q = 0; q < PM; ++q) idx[q] = q;
        g_row = scores + (size_t)p * PM;
        qsort(idx, (size_t)PM, sizeof(int), cmp_desc);
        for (int r = 0; r < R; ++r) topk[(size_t)p * R + r] = idx[r];
    }
    free(idx);
    return 0;
}
