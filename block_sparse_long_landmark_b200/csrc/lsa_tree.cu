// lsa_tree.cu -- tree variant of the clustered index: a hierarchy over the
// flat index's clusters and a beam search down it.
//
// The Latent Sparse Attention post, section "Индекс перестаёт перебирать
// весь контекст": the clusters are grouped into a hierarchy that a query
// walks keeping a few good branches per level, so it is compared against far
// fewer centres than a flat scan of every cluster.  Reading (the post gives
// no construction): the flat clusters are the leaves; every level above is a
// Ward clustering of the level below into ceil(n / fanout) nodes, each node
// weighted by the key positions it holds, numbered by their first child; a
// node's centre is the mass-weighted mean of its children's centres.  The
// search keeps the `beam` best nodes of a level by (score desc, id asc),
// descends into their children, and at the leaves keeps the `top_clusters`
// best, which are then expanded to key positions exactly as in the flat decode.
//
// Build: one CTA per (batch, kv-head), level by level.  Ward's merges run in
// fp64 with a cached nearest neighbour per node: the all-pairs start stages
// 32-row tiles in shared memory; after each merge only the costs to the
// merged node are recomputed (a node whose neighbour was one of the two
// merged nodes is rescanned).  Every distance is summed in one fixed order
// (lane l takes elements l, l + 32, ... in turn, then the lanes are added
// 16 apart, 8 apart, ..., 1 apart), whichever kernel step computes it, so
// the cost of a pair is the same number wherever it is compared.
#include <math_constants.h>

#include "common.cuh"
#include "lsa.cuh"
#include "lsa_dev.cuh"

namespace sa {
namespace {

struct TreeArgs {
    LsaShape s;
    LsaTreePlan tp;
    const double *centres;     // index centres [B*Hkv][C][d] (the leaves)
    const int32_t *sizes;      // index cluster sizes in items [B*Hkv][C]
    unsigned char *tree;       // tree buffer (layout of tp)
    double *W;                 // build workspace: working centres [B*Hkv][n0][d]
};

__device__ __forceinline__ double *lvl_cent(const TreeArgs &a, int lv) {
    return reinterpret_cast<double *>(a.tree + a.tp.off_cent[lv]);
}
__device__ __forceinline__ double *lvl_mass(const TreeArgs &a, int lv) {
    return reinterpret_cast<double *>(a.tree + a.tp.off_mass[lv]);
}
__device__ __forceinline__ int32_t *lvl_cs(const TreeArgs &a, int lv) {
    return reinterpret_cast<int32_t *>(a.tree + a.tp.off_cs[lv]);
}
__device__ __forceinline__ int32_t *lvl_ci(const TreeArgs &a, int lv) {
    return reinterpret_cast<int32_t *>(a.tree + a.tp.off_ci[lv]);
}

// 32 per-lane partial sums (one per value) -> lane l returns the total of
// value l, combined over the lanes 16 apart, then 8, 4, 2, 1 apart: the same
// tree (and, addition being commutative, the same bits) as warp_total below.
__device__ __forceinline__ double reduce_scatter32(double (&v)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const bool up = lane & o;
#pragma unroll
        for (int x = 0; x < o; ++x) {
            const double send = up ? v[x] : v[x + o];
            const double keep = up ? v[x + o] : v[x];
            v[x] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0];
}
__device__ __forceinline__ double warp_total(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Ward's increase of the within-cluster sum of squares for clusters of mass
// mi and mj whose centres are `dist` apart (squared), in the oracle's order.
__device__ __forceinline__ double ward_cost(double mi, double mj, double dist) {
    return __dmul_rn(__ddiv_rn(__dmul_rn(mi, mj), __dadd_rn(mi, mj)), dist);
}

// (cost, id) order: lower cost first, then lower id
__device__ __forceinline__ bool better(double c, int i, double bc, int bi) {
    return c < bc || (c == bc && i < bi);
}

// Warp-wide minimum of (cost, id); every lane gets it.
__device__ __forceinline__ void warp_min(double &c, int &i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double oc = __shfl_xor_sync(0xffffffffu, c, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (better(oc, oi, c, i)) {
            c = oc;
            i = oi;
        }
    }
}

constexpr int kTileRows = 32;

template <int D>
__global__ void __launch_bounds__(kLsaThreads) lsa_tree_build_kernel(TreeArgs a) {
    constexpr int EPL = D / 32;                    // elements per lane: lane, lane + 32, ...
    constexpr int NW = kLsaThreads / 32;
    extern __shared__ __align__(16) unsigned char smraw[];
    const LsaShape &s = a.s;
    const LsaTreePlan &tp = a.tp;
    const int n0 = tp.n[0];
    double *tile = reinterpret_cast<double *>(smraw);         // [32][D]
    double *wm = tile + kTileRows * D;                         // [n0] masses of the live clusters
    double *nnc = wm + n0;                                     // [n0] cost to the nearest neighbour
    int *nn = reinterpret_cast<int *>(nnc + n0);               // [n0] nearest neighbour
    int *owner = nn + n0;                                      // [n0] cluster (its first node) of node x
    int *alive = owner + n0;                                   // [n0]
    int *flist = alive + n0;                                   // [n0] nodes to rescan / ranks
    __shared__ double rc[NW];
    __shared__ int rix[NW], nflag, pick[2];
    __shared__ int red[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bg = blockIdx.x;

    // leaf masses: the key positions each cluster holds
    {
        double *m0 = lvl_mass(a, 0) + (size_t)bg * n0;
        const int32_t *sz = a.sizes + (size_t)bg * s.ctotal;
        for (int c = tid; c < n0; c += kLsaThreads) m0[c] = (double)min(max(sz[c], 0), s.seg) * (double)s.pool;
    }
    __syncthreads();
    double *W = a.W + (size_t)bg * n0 * D;
    for (int lv = 1; lv < tp.L; ++lv) {
        const int n = tp.n[lv - 1], k = tp.n[lv];
        const double *X = (lv == 1 ? a.centres : lvl_cent(a, lv - 1)) + (size_t)bg * n * D;
        const double *M = lvl_mass(a, lv - 1) + (size_t)bg * n;
        for (int x = tid; x < n * D; x += kLsaThreads) W[x] = X[x];
        for (int i = tid; i < n; i += kLsaThreads) {
            wm[i] = M[i];
            owner[i] = i;
            alive[i] = 1;
        }
        __syncthreads();
        // ---- nearest neighbour of every node: all pairs, 32-row tiles -------
        for (int i0 = 0; i0 < n; i0 += NW * 4) {
            double xi[4][EPL], best[4];
            int bj[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int i = min(i0 + warp * 4 + r, n - 1);
#pragma unroll
                for (int t = 0; t < EPL; ++t) xi[r][t] = W[(size_t)i * D + lane + 32 * t];
                best[r] = CUDART_INF;
                bj[r] = 0x7fffffff;
            }
            for (int j0 = 0; j0 < n; j0 += kTileRows) {
                __syncthreads();
                for (int x = tid; x < kTileRows * D; x += kLsaThreads) {
                    const int j = j0 + x / D;
                    tile[x] = j < n ? W[(size_t)j * D + x % D] : 0.0;
                }
                __syncthreads();
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    double v[32];
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        double acc = 0.0;
#pragma unroll
                        for (int t = 0; t < EPL; ++t) {
                            const double df = xi[r][t] - tile[jj * D + lane + 32 * t];
                            acc = fma(df, df, acc);
                        }
                        v[jj] = acc;
                    }
                    const double dist = reduce_scatter32(v);
                    const int i = i0 + warp * 4 + r, j = j0 + lane;
                    if (i < n && j < n && j != i) {
                        const double c = ward_cost(wm[i], wm[j], dist);
                        if (better(c, j, best[r], bj[r])) {
                            best[r] = c;
                            bj[r] = j;
                        }
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                warp_min(best[r], bj[r]);
                const int i = i0 + warp * 4 + r;
                if (lane == 0 && i < n) {
                    nn[i] = bj[r];
                    nnc[i] = best[r];
                }
            }
        }
        __syncthreads();
        // ---- merges -----------------------------------------------------------
        for (int live = n; live > k; --live) {
            // (1) the cheapest pair: the lowest node whose neighbour cost is the
            // minimum, with its neighbour (the lowest partner at that cost)
            double c = CUDART_INF;
            int ci = 0x7fffffff;
            for (int i = tid; i < n; i += kLsaThreads)
                if (alive[i] && better(nnc[i], i, c, ci)) {
                    c = nnc[i];
                    ci = i;
                }
            warp_min(c, ci);
            if (lane == 0) {
                rc[warp] = c;
                rix[warp] = ci;
            }
            if (tid == 0) nflag = 0;
            __syncthreads();
            if (tid == 0) {
                double bc = rc[0];
                int bi = rix[0];
                for (int w = 1; w < NW; ++w)
                    if (better(rc[w], rix[w], bc, bi)) {
                        bc = rc[w];
                        bi = rix[w];
                    }
                pick[0] = bi;
                pick[1] = (bi >= 0 && bi < n) ? nn[bi] : -1;
            }
            __syncthreads();
            const int pa = pick[0], pb = pick[1];
            if (pa < 0 || pa >= n || pb < 0 || pb >= n || pa == pb || !alive[pa] || !alive[pb]) break;   // cannot happen
            const int ma = min(pa, pb), mb = max(pa, pb);   // the merged cluster keeps the lower id
            // (2) merge mb into ma: centre (m_a c_a + m_b c_b) / (m_a + m_b), as the oracle rounds it
            const double na = wm[ma], nb = wm[mb];
            for (int e = tid; e < D; e += kLsaThreads)
                W[(size_t)ma * D + e] = __ddiv_rn(__dadd_rn(__dmul_rn(na, W[(size_t)ma * D + e]),
                                                            __dmul_rn(nb, W[(size_t)mb * D + e])),
                                                  __dadd_rn(na, nb));
            for (int x = tid; x < n; x += kLsaThreads)
                if (owner[x] == mb) owner[x] = ma;
            __syncthreads();
            if (tid == 0) {
                wm[ma] = __dadd_rn(na, nb);
                alive[mb] = 0;
            }
            __syncthreads();
            // (3) costs to the merged node: update neighbours, flag nodes whose
            // neighbour was one of the merged two, and find the merged node's own
            double xa[EPL];
#pragma unroll
            for (int t = 0; t < EPL; ++t) xa[t] = W[(size_t)ma * D + lane + 32 * t];
            double bc = CUDART_INF;
            int bi = 0x7fffffff;
            for (int i0 = warp * 32; i0 < n; i0 += NW * 32) {
                double v[32];
#pragma unroll
                for (int ii = 0; ii < 32; ++ii) {
                    const int i = min(i0 + ii, n - 1);
                    double acc = 0.0;
#pragma unroll
                    for (int t = 0; t < EPL; ++t) {
                        const double df = W[(size_t)i * D + lane + 32 * t] - xa[t];
                        acc = fma(df, df, acc);
                    }
                    v[ii] = acc;
                }
                const double dist = reduce_scatter32(v);
                const int i = i0 + lane;
                if (i < n && alive[i] && i != ma) {
                    const double cc = ward_cost(wm[i], wm[ma], dist);
                    if (better(cc, i, bc, bi)) {
                        bc = cc;
                        bi = i;
                    }
                    if (nn[i] == ma || nn[i] == mb) {
                        flist[atomicAdd(&nflag, 1)] = i;
                    } else if (better(cc, ma, nnc[i], nn[i])) {
                        nn[i] = ma;
                        nnc[i] = cc;
                    }
                }
            }
            warp_min(bc, bi);
            __syncthreads();
            if (lane == 0) {
                rc[warp] = bc;
                rix[warp] = bi;
            }
            __syncthreads();
            if (tid == 0) {
                double b2 = rc[0];
                int i2 = rix[0];
                for (int w = 1; w < NW; ++w)
                    if (better(rc[w], rix[w], b2, i2)) {
                        b2 = rc[w];
                        i2 = rix[w];
                    }
                nn[ma] = i2;
                nnc[ma] = b2;
            }
            __syncthreads();
            // (4) rescan the flagged nodes against every live node
            const int nf = nflag;
            for (int f = 0; f < nf; ++f) {
                const int x = flist[f];
                double xf[EPL];
#pragma unroll
                for (int t = 0; t < EPL; ++t) xf[t] = W[(size_t)x * D + lane + 32 * t];
                double fc = CUDART_INF;
                int fi = 0x7fffffff;
                for (int j0 = warp * 32; j0 < n; j0 += NW * 32) {
                    double v[32];
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int j = min(j0 + jj, n - 1);
                        double acc = 0.0;
#pragma unroll
                        for (int t = 0; t < EPL; ++t) {
                            const double df = xf[t] - W[(size_t)j * D + lane + 32 * t];
                            acc = fma(df, df, acc);
                        }
                        v[jj] = acc;
                    }
                    const double dist = reduce_scatter32(v);
                    const int j = j0 + lane;
                    if (j < n && alive[j] && j != x) {
                        const double cc = ward_cost(wm[x], wm[j], dist);
                        if (better(cc, j, fc, fi)) {
                            fc = cc;
                            fi = j;
                        }
                    }
                }
                warp_min(fc, fi);
                if (lane == 0) {
                    rc[warp] = fc;
                    rix[warp] = fi;
                }
                __syncthreads();
                if (tid == 0) {
                    double b2 = rc[0];
                    int i2 = rix[0];
                    for (int w = 1; w < NW; ++w)
                        if (better(rc[w], rix[w], b2, i2)) {
                            b2 = rc[w];
                            i2 = rix[w];
                        }
                    nn[x] = i2;
                    nnc[x] = b2;
                }
                __syncthreads();
            }
        }
        // ---- the level: parents numbered by their first child ------------------
        // rank of every live cluster among the live ones (reusing flist)
        int carry = 0;
        for (int i0 = 0; i0 < n; i0 += kLsaThreads) {
            const int i = i0 + tid;
            const int f = (i < n && alive[i]) ? 1 : 0;
            int tot;
            const int incl = block_scan_incl(f, red, &tot);
            if (i < n) flist[i] = carry + incl - f;
            carry += tot;
        }
        __syncthreads();
        int32_t *cs = lvl_cs(a, lv) + (size_t)bg * (k + 1);
        int32_t *ci = lvl_ci(a, lv) + (size_t)bg * n;
        double *cent = lvl_cent(a, lv) + (size_t)bg * k * D;
        double *mass = lvl_mass(a, lv) + (size_t)bg * k;
        // children per parent (nnc reused as int counters), then their starts
        int *cntp = reinterpret_cast<int *>(nnc);
        for (int p = tid; p < k; p += kLsaThreads) cntp[p] = 0;
        __syncthreads();
        for (int x = tid; x < n; x += kLsaThreads) atomicAdd(&cntp[flist[owner[x]]], 1);
        __syncthreads();
        carry = 0;
        for (int p0 = 0; p0 < k; p0 += kLsaThreads) {
            const int p = p0 + tid;
            const int v = p < k ? cntp[p] : 0;
            int tot;
            const int incl = block_scan_incl(v, red, &tot);
            if (p < k) {
                cs[p] = carry + incl - v;
                cntp[p] = carry + incl - v;          // cursor
            }
            carry += tot;
        }
        if (tid == 0) cs[k] = carry;
        __syncthreads();
        // children ascending within each parent: one warp walks the nodes in order
        if (warp == 0) {
            for (int x0 = 0; x0 < n; x0 += 32) {
                const int x = x0 + lane;
                const int p = x < n ? flist[owner[x]] : -1;
                const unsigned act = __ballot_sync(0xffffffffu, x < n);
                if (x < n) {
                    const unsigned same = __match_any_sync(act, p);
                    const int before = __popc(same & ((1u << lane) - 1u));
                    ci[cntp[p] + before] = x;
                    __syncwarp(same);
                    if (before == 0) cntp[p] += __popc(same);
                }
                __syncwarp();
            }
        }
        __syncthreads();
        // centres and masses: the children's mass-weighted mean, summed in child order
        for (int p = warp; p < k; p += NW) {
            const int c0 = cs[p], c1 = cs[p + 1];
            double msum = 0.0;
            for (int c = c0; c < c1; ++c) msum = __dadd_rn(msum, M[ci[c]]);
            for (int e = lane; e < D; e += 32) {
                double acc = 0.0;
                for (int c = c0; c < c1; ++c) {
                    const int x = ci[c];
                    const double t = __dmul_rn(M[x], X[(size_t)x * D + e]);
                    acc = c == c0 ? t : __dadd_rn(acc, t);
                }
                cent[(size_t)p * D + e] = __ddiv_rn(acc, msum);
            }
            if (lane == 0) mass[p] = msum;
        }
        __syncthreads();
    }
}

// Beam search of one (batch, kv-head): the pooled query scored against the
// top level's nodes, the `beam` best of each level expanded into their
// children, the `top_clusters` best leaves expanded to key positions.
struct TreeSelArgs {
    LsaDecArgs d;
    LsaTreePlan tp;
    const unsigned char *tree;
    int beam;
    int32_t *compared;     // optional [B*Hkv]
};

template <typename T>
__global__ void __launch_bounds__(kLsaThreads) lsa_tree_select_kernel(TreeSelArgs ta) {
    extern __shared__ __align__(16) unsigned char smraw[];
    const LsaDecArgs &a = ta.d;
    const LsaShape &s = a.s;
    const LsaTreePlan &tp = ta.tp;
    const int F = tp.maxfront;
    double *qbar = reinterpret_cast<double *>(smraw);                 // [d]
    int *red = reinterpret_cast<int *>(qbar + s.d);                   // [8]
    int *misc = red + 8;                                              // [8]
    int *hist = misc + 8;                                             // [264]
    uint64_t *keys = reinterpret_cast<uint64_t *>(hist + 264);        // [F]
    int *fr = reinterpret_cast<int *>(keys + F);                      // [F] frontier, ascending ids
    int *pos = fr + F;                                                // [F]
    int *mark = pos + F;                                              // [F]
    int *off = mark + F;                                              // [F + 1]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bg = blockIdx.x, b = bg / s.Hkv, g = bg % s.Hkv;
    const int D = s.d;
    const T *q = (const T *)a.q;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the attention may start early
    for (int e = tid; e < D; e += kLsaThreads) {
        double acc = 0.0;
        for (int h = 0; h < s.G; ++h) acc += (double)to_f(q[((size_t)b * s.Hq + g * s.G + h) * D + e]);
        qbar[e] = acc / s.G;
    }
    const int top = tp.L - 1;
    int nf = tp.n[top];
    for (int i = tid; i < nf; i += kLsaThreads) fr[i] = i;
    __syncthreads();
    int compared = 0;
    bool nan_seen = false;
    for (int lv = top; lv >= 0; --lv) {
        const double *cen = lv == 0 ? a.centres + (size_t)bg * s.ctotal * D
                                    : reinterpret_cast<const double *>(ta.tree + tp.off_cent[lv]) +
                                          (size_t)bg * tp.n[lv] * D;
        // a warp per centre, four centres of the frontier in flight per warp
        for (int i0 = warp * 4; i0 < nf; i0 += 4 * (kLsaThreads / 32)) {
            double part[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const double *row = cen + (size_t)fr[min(i0 + u, nf - 1)] * D;
                double acc = 0.0;
                for (int e = lane; e < D; e += 32) acc = fma(row[e], qbar[e], acc);
                part[u] = acc;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const double acc = warp_total(part[u]);
                if (lane == 0 && i0 + u < nf) {
                    const double sc = (double)s.scale * acc;
                    nan_seen |= isnan(sc);
                    keys[i0 + u] = ord_key64(sc);
                }
            }
        }
        compared += nf;
        __syncthreads();
        const int keep = lv > 0 ? ta.beam : min(s.top_clusters, s.ctotal);
        const int nk = block_topk64(keys, nf, keep, pos, hist, red);
        if (lv == 0) {
            // the chosen leaves (ascending ids) go to the position expansion; `mark` holds them
            for (int i = tid; i < nk; i += kLsaThreads) mark[i] = fr[pos[i]];
            __syncthreads();
            expand_positions(a, bg, mark, nk, off, red);
            break;
        }
        // next frontier: the children of the kept nodes, in ascending id order
        const int nb = tp.n[lv - 1];
        const int32_t *cs = reinterpret_cast<const int32_t *>(ta.tree + tp.off_cs[lv]) + (size_t)bg * (tp.n[lv] + 1);
        const int32_t *ci = reinterpret_cast<const int32_t *>(ta.tree + tp.off_ci[lv]) + (size_t)bg * nb;
        if (nk <= kLsaThreads) {
            // few kept nodes: gather their children, then place each by its rank
            int c0 = 0, cn = 0;
            if (tid < nk) {
                const int p = fr[pos[tid]];
                c0 = cs[p];
                cn = max(0, cs[p + 1] - c0);
            }
            int nc;
            const int at = block_scan_incl(cn, red, &nc) - cn;
            if (nc <= min(kLsaThreads, F)) {
                for (int c = 0; c < cn; ++c) {
                    const int x = ci[c0 + c];
                    mark[at + c] = (x >= 0 && x < nb) ? x : -1;
                }
                __syncthreads();
                int x = -1, r = 0;
                if (tid < nc) {
                    x = mark[tid];
                    for (int j = 0; j < nc; ++j) {
                        const int y = mark[j];
                        r += y >= 0 && (y < x || (y == x && j < tid));
                    }
                }
                int nv;
                block_scan_incl(x >= 0 ? 1 : 0, red, &nv);
                if (x >= 0) fr[r] = x;
                nf = nv;
                __syncthreads();
                continue;
            }
        }
        for (int x = tid; x < nb; x += kLsaThreads) mark[x] = 0;
        __syncthreads();
        for (int i = warp; i < nk; i += kLsaThreads / 32) {
            const int p = fr[pos[i]];
            for (int c = cs[p] + lane; c < cs[p + 1]; c += 32) {
                const int x = ci[c];
                if (x >= 0 && x < nb) mark[x] = 1;
            }
        }
        __syncthreads();
        int carry = 0;
        for (int x0 = 0; x0 < nb; x0 += kLsaThreads) {
            const int x = x0 + tid;
            const int f = x < nb ? mark[x] : 0;
            int tot;
            const int at = block_scan_incl(f, red, &tot) - f;
            if (f) fr[carry + at] = x;
            carry += tot;
        }
        nf = carry;
        __syncthreads();
    }
    if (nan_seen) set_status(a.status, kStatusNaN);
    if (tid == 0 && ta.compared) ta.compared[bg] = compared;
}

}  // namespace

bool lsa_tree_plan(const LsaShape &s, int fanout, LsaTreePlan &tp) {
    if (fanout < 2 || fanout > 64) return false;
    const int n0 = s.ctotal;
    if (n0 < 1 || n0 > kLsaTreeMaxLeaves) return false;
    tp.L = 1;
    tp.n[0] = n0;
    while (tp.n[tp.L - 1] > fanout) {
        if (tp.L == kLsaMaxLevels) return false;
        tp.n[tp.L] = (tp.n[tp.L - 1] + fanout - 1) / fanout;
        ++tp.L;
    }
    tp.maxfront = n0;
    const size_t bgs = (size_t)s.B * s.Hkv;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    size_t off = 0;
    for (int lv = 0; lv < tp.L; ++lv) {
        tp.off_mass[lv] = off;
        off += al(bgs * tp.n[lv] * 8);
        if (lv == 0) {
            tp.off_cent[0] = tp.off_cs[0] = tp.off_ci[0] = 0;   // the leaves are the index's clusters
            continue;
        }
        tp.off_cent[lv] = off;
        off += al(bgs * tp.n[lv] * s.d * 8);
        tp.off_cs[lv] = off;
        off += al(bgs * (tp.n[lv] + 1) * 4);
        tp.off_ci[lv] = off;
        off += al(bgs * tp.n[lv - 1] * 4);
    }
    tp.bytes = off;
    tp.work_bytes = al(bgs * n0 * s.d * 8);
    return true;
}

static size_t tree_build_smem(const LsaShape &s, const LsaTreePlan &tp) {
    return (size_t)kTileRows * s.d * 8 + (size_t)tp.n[0] * (8 + 8 + 4 * 4);
}

static size_t tree_select_smem(const LsaShape &s, const LsaTreePlan &tp) {
    return (size_t)s.d * 8 + (8 + 8 + 264) * 4 + (size_t)tp.maxfront * (8 + 4 + 4 + 4 + 4) + 4;
}

cudaError_t launch_lsa_tree_build(const LsaShape &s, const LsaTreePlan &tp, const double *centres,
                                  const int32_t *sizes, void *tree, double *work, cudaStream_t st) {
    TreeArgs a{};
    a.s = s;
    a.tp = tp;
    a.centres = centres;
    a.sizes = sizes;
    a.tree = static_cast<unsigned char *>(tree);
    a.W = work;
    const size_t smem = tree_build_smem(s, tp);
    void (*kern)(TreeArgs) = s.d == 128 ? lsa_tree_build_kernel<128> : lsa_tree_build_kernel<64>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(s.B * s.Hkv), kLsaThreads, smem, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_lsa_tree_decode(const LsaShape &s, const LsaDecPlan &pl, const LsaTreePlan &tp, int beam,
                                   const void *q, const void *K, const void *V, const double *centres,
                                   const int32_t *members, const int32_t *sizes, const void *tree, void *ws, void *o,
                                   float *lse, int32_t *kept, int32_t *compared, cudaStream_t st) {
    TreeSelArgs ta{};
    LsaDecArgs &a = ta.d;
    a.s = s;
    a.pl = pl;
    a.q = q;
    a.K = K;
    a.V = V;
    a.centres = centres;
    a.members = members;
    a.sizes = sizes;
    a.o = o;
    a.lse = lse;
    a.kept = kept;
    lsa_bind_workspace(a, ws);
    ta.tp = tp;
    ta.tree = static_cast<const unsigned char *>(tree);
    ta.beam = beam;
    ta.compared = compared;
    const size_t smem = tree_select_smem(s, tp);
    void (*kern)(TreeSelArgs) =
        s.dtype == SA_BF16 ? lsa_tree_select_kernel<__nv_bfloat16> : lsa_tree_select_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(s.B * s.Hkv), kLsaThreads, smem, st>>>(ta);
    note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_lsa_attend(a, st);
}

}  // namespace sa
