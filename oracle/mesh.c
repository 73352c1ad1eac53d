/*
 * Oracle (test infrastructure only): geodesic farthest-point sampling and
 * nearest-centre patches on a triangle-mesh graph, plain fp64 on the CPU.
 * Only tests/, the smoke check and the bench's CPU baseline may load this; it
 * shares no code with the CUDA path.
 *
 * Source: ai4snews digest of "Spatial-Spectral Coupling as Attention",
 * "Interpretation" (the surface is partitioned with geodesic farthest-point
 * sampling) and the project page, "Geo-FlashAttention" (partition each
 * surface into geodesic patches).  The pages name no geodesic solver; on a
 * mesh the plainest reading is the shortest-path distance along mesh edges.
 *
 * Readings taken where the pages are silent:
 *  - the mesh is a graph: vertices, undirected edges with non-negative fp64
 *    lengths (the caller's; the synthetic meshes use Euclidean edge lengths);
 *  - the distance of a path is its edge lengths added in fp64 from the
 *    source outward, d(v) = min over paths of that sum (Dijkstra's value);
 *  - FPS starts at the seed; each next centre is the vertex whose distance to
 *    the nearest chosen centre is largest, ties to the lowest vertex index
 *    (a vertex no centre reaches has distance +inf, so every connected part
 *    of the mesh receives a centre before a second one in any part);
 *  - the patch of a vertex is its nearest centre, ties to the lowest patch
 *    index (a later centre takes a vertex only when strictly nearer); a
 *    vertex that no centre reaches (fewer centres than connected parts) has
 *    no patch, owner -1.
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared (see oracle/build.py).
 */
#include <math.h>
#include <stdlib.h>

/* binary min-heap of (distance, vertex) entries; stale entries are skipped */
typedef struct {
    double d;
    int v;
} Entry;

static void heap_push(Entry* h, long* size, Entry e) {
    long i = (*size)++;
    while (i > 0) {
        long p = (i - 1) / 2;
        if (h[p].d <= e.d) break;
        h[i] = h[p];
        i = p;
    }
    h[i] = e;
}

static Entry heap_pop(Entry* h, long* size) {
    Entry top = h[0];
    Entry last = h[--(*size)];
    long i = 0;
    for (;;) {
        long l = 2 * i + 1, r = l + 1, m = i;
        double dm = last.d;
        if (l < *size && h[l].d < dm) { m = l; dm = h[l].d; }
        if (r < *size && h[r].d < dm) { m = r; }
        if (m == i) break;
        h[i] = h[m];
        i = m;
    }
    if (*size > 0) h[i] = last;
    return top;
}

/* Single-source shortest paths from s: dist [n] receives d(s, v) (+inf when
 * unreachable).  heap has room for nnz + 1 entries.  Edges with a negative or
 * NaN length or an endpoint out of range are skipped.  Returns the number of
 * skipped edge visits. */
static long dijkstra(const int* off, const int* adj, const double* w, int n, int s, double* dist,
                     Entry* heap) {
    long skipped = 0, size = 0;
    for (int v = 0; v < n; ++v) dist[v] = INFINITY;
    dist[s] = 0.0;
    heap_push(heap, &size, (Entry){0.0, s});
    while (size > 0) {
        Entry e = heap_pop(heap, &size);
        if (e.d > dist[e.v]) continue; /* stale */
        for (int k = off[e.v]; k < off[e.v + 1]; ++k) {
            int u = adj[k];
            double wk = w[k];
            if (u < 0 || u >= n || !(wk >= 0.0)) { ++skipped; continue; }
            double nd = e.d + wk;
            if (nd < dist[u]) {
                dist[u] = nd;
                heap_push(heap, &size, (Entry){nd, u});
            }
        }
    }
    return skipped;
}

/* Geodesic FPS plus nearest-centre assignment on the graph (off [n+1], adj
 * [nnz], w [nnz]).  centers [P]; owner [n]; dist_out [n] (nullable) receives
 * every vertex's final distance to its nearest centre.  Returns 0, -1 on bad
 * arguments, -2 when allocation fails, or the count of skipped edges (> 0)
 * when the graph holds invalid edges (results then computed without them). */
long oracle_fps_mesh(const int* off, const int* adj, const double* w, int n, int P, int seed,
                     int* centers, int* owner, double* dist_out) {
    if (n < 1 || P < 1 || P > n || seed < 0 || seed >= n || off[0] != 0) return -1;
    for (int v = 0; v < n; ++v)
        if (off[v + 1] < off[v]) return -1;
    const long nnz = off[n];
    double* best = (double*)malloc(sizeof(double) * (size_t)n);
    double* d = (double*)malloc(sizeof(double) * (size_t)n);
    Entry* heap = (Entry*)malloc(sizeof(Entry) * (size_t)(nnz + 1));
    if (!best || !d || !heap) { free(best); free(d); free(heap); return -2; }
    for (int v = 0; v < n; ++v) { best[v] = INFINITY; owner[v] = -1; }
    long skipped = 0;
    int c = seed;
    for (int t = 0; t < P; ++t) {
        centers[t] = c;
        skipped += dijkstra(off, adj, w, n, c, d, heap);
        for (int v = 0; v < n; ++v)
            if (d[v] < best[v]) { best[v] = d[v]; owner[v] = t; }
        /* next centre: the largest distance, ties to the lowest index */
        int arg = 0;
        for (int v = 1; v < n; ++v)
            if (best[v] > best[arg]) arg = v;
        c = arg;
    }
    if (dist_out)
        for (int v = 0; v < n; ++v) dist_out[v] = best[v];
    free(best); free(d); free(heap);
    return skipped > 0 ? skipped / (P > 0 ? P : 1) + 1 : 0;
}

/* d(s, v) for one source (the single-source distances FPS is built from). */
long oracle_sssp(const int* off, const int* adj, const double* w, int n, int s, double* dist) {
    if (n < 1 || s < 0 || s >= n) return -1;
    Entry* heap = (Entry*)malloc(sizeof(Entry) * (size_t)(off[n] + 1));
    if (!heap) return -2;
    long sk = dijkstra(off, adj, w, n, s, dist, heap);
    free(heap);
    return sk;
}
