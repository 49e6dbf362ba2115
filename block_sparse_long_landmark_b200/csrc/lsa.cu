// lsa.cu -- flat clustered index of Latent Sparse Attention (decode).
//
// The Latent Sparse Attention post, section "Индекс перестаёт перебирать
// весь контекст": adjacent keys are pooled into items; once a segment of
// items is complete it is clustered by Ward's method and frozen; the index
// keeps each cluster's centre and the positions of its items.  A query is
// scored against every centre (flat variant), the best clusters are expanded
// back to positions, the context start and a recent window are added, and the
// query attends to that set.
//
// Kernel 1 (build): one CTA per (batch, kv-head, complete segment).  Items
// (means of `pool` keys) and Ward's merges in double precision -- the merge
// order is a chain of exact comparisons, taken in the precision the index's
// definition is written in -- down to `clusters` clusters per segment; writes
// each cluster's centre and its item ids.
// Kernel 2 (decode): one CTA per (batch, kv-head).  Pooled query of the
// group's heads; scores of every centre (double); the best `top_clusters` by
// (score desc, cluster id asc); a bitmap of kept positions (sink, window,
// chosen clusters' items); then one warp per query head runs an fp32 online
// softmax over the kept positions.
#include <math_constants.h>

#include "common.cuh"
#include "lsa.cuh"
#include "bounds.cuh"
#include "lsa_dev.cuh"

namespace sa {
namespace {


template <typename T>
__global__ void __launch_bounds__(kLsaThreads) lsa_build_kernel(LsaShape s, const void *Kv, double *centres64,
                                                               int32_t *members, int32_t *msize) {
    extern __shared__ double sm[];
    const int D = s.d, S = s.seg;
    double *cent = sm;                                   // [S][D] cluster centres (item means at start)
    double *cost = cent + S * D;                         // [kLsaThreads] per-thread best cost
    int *csize = reinterpret_cast<int *>(cost + kLsaThreads);   // [S]
    int *owner = csize + S;                              // [S] item -> cluster id (its first item's slot)
    int *alive = owner + S;                              // [S]
    int *bpair = alive + S;                              // [kLsaThreads] per-thread best pair
    const int tid = threadIdx.x;
    const int sg = blockIdx.x % s.nseg, bg = blockIdx.x / s.nseg;
    const T *K = (const T *)Kv + (size_t)bg * s.N * D;
    // items of this segment
    for (int x = tid; x < S * D; x += kLsaThreads) {
        const int i = x / D, e = x % D;
        const int t0 = (sg * S + i) * s.pool;
        double acc = 0.0;
        for (int t = 0; t < s.pool; ++t) acc += (double)to_f(K[(size_t)(t0 + t) * D + e]);
        cent[x] = acc / s.pool;
    }
    for (int i = tid; i < S; i += kLsaThreads) {
        csize[i] = 1;
        owner[i] = i;
        alive[i] = 1;
    }
    __syncthreads();
    const int npairs = S * (S - 1) / 2;
    for (int live = S; live > s.clusters; --live) {
        // every thread: its best alive pair (a < b) by (cost, a, b)
        double best = CUDART_INF;
        int bp = 0x7fffffff;
        for (int p = tid; p < npairs; p += kLsaThreads) {
            // pair index -> (a, b), a < b, in row-major order of a
            int a = 0, rem = p;
            while (rem >= S - 1 - a) { rem -= S - 1 - a; ++a; }
            const int b = a + 1 + rem;
            if (!alive[a] || !alive[b]) continue;
            double dist = 0.0;
            for (int e = 0; e < D; ++e) {
                const double df = cent[a * D + e] - cent[b * D + e];
                dist += df * df;
            }
            const double na = csize[a], nb = csize[b];
            double c = na * nb / (na + nb) * dist;
            if (!(c <= CUDART_INF)) c = CUDART_INF;      // NaN ranks as +inf: some alive pair always wins
            const int code = a * S + b;
            if (c < best || (c == best && code < bp)) { best = c; bp = code; }
        }
        cost[tid] = best;
        bpair[tid] = bp;
        __syncthreads();
        for (int w = kLsaThreads / 2; w > 0; w >>= 1) {
            if (tid < w) {
                const double c2 = cost[tid + w];
                const int p2 = bpair[tid + w];
                if (c2 < cost[tid] || (c2 == cost[tid] && p2 < bpair[tid])) {
                    cost[tid] = c2;
                    bpair[tid] = p2;
                }
            }
            __syncthreads();
        }
        const int bp0 = bpair[0];
        if (bp0 < 0 || bp0 >= S * S) break;              // no alive pair (cannot happen while live >= 2)
        const int a = bp0 / S, b = bp0 % S;
        const double na = csize[a], nb = csize[b];
        __syncthreads();
        for (int e = tid; e < D; e += kLsaThreads) cent[a * D + e] = (na * cent[a * D + e] + nb * cent[b * D + e]) / (na + nb);
        for (int i = tid; i < S; i += kLsaThreads)
            if (owner[i] == b) owner[i] = a;
        if (tid == 0) {
            csize[a] += csize[b];
            alive[b] = 0;
        }
        __syncthreads();
    }
    // clusters numbered by their first item (surviving ids are first items)
    if (tid == 0) {
        int c = 0;
        for (int i = 0; i < S; ++i) {
            if (!alive[i]) continue;
            const size_t cid = ((size_t)bg * s.nseg + sg) * s.clusters + c;
            int m = 0;
            for (int x = 0; x < S; ++x)
                if (owner[x] == i) members[cid * S + m++] = sg * S + x;
            for (int x = m; x < S; ++x) members[cid * S + x] = -1;
            msize[cid] = m;
            alive[i] = 1000 + c;          // remember the output slot
            ++c;
        }
    }
    __syncthreads();
    for (int i = 0; i < S; ++i) {
        if (alive[i] < 1000) continue;
        const size_t cid = ((size_t)bg * s.nseg + sg) * s.clusters + (alive[i] - 1000);
        for (int e = tid; e < D; e += kLsaThreads) centres64[cid * D + e] = cent[i * D + e];
    }
}

// ---------------------------------------------------------------------------
// Decode through the index
// ---------------------------------------------------------------------------

// Kernel 2 (flat decode, step 1): one CTA per (batch, kv-head, chunk of
// centres).  Pooled query of the kv-group's heads (fp64), score of every
// centre of the chunk, scale * <q, centre> in fp64; the chunk passes all its
// scores to the merge, or, when the merge could not hold every centre, its
// best kk by (score desc, id asc).  The last chunk CTA of a (batch, kv-head)
// takes the top_clusters best of the candidates with a block-wide radix
// select and expands them into the flat list of kept key positions.
// The kw-th largest (1 <= kw <= 32) of the 32 lanes' 64-bit values: each
// lane ranks its value against every lane's (equal values in lane order).
__device__ __forceinline__ uint64_t warp_kth_largest64(uint64_t v, int kw) {
    const int lane = threadIdx.x & 31;
    int rk = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const uint64_t x = __shfl_sync(0xffffffffu, v, j);
        rk += (x > v) | ((x == v) & (j < lane));
    }
    const unsigned at = __ballot_sync(0xffffffffu, rk == kw - 1);
    return __shfl_sync(0xffffffffu, v, __ffs(at) - 1);
}

// The merge's top-k (k <= 256) of keys[0..n) (n <= 16 * threads): a lower
// bound L of the k-th largest key (warp w's ceil(k/8)-th largest lane
// maximum, the least over the warps, so that at least k keys are >= L), the
// keys >= L and their ids copied in list order into `scratch` (1536 ints,
// 8-byte aligned), ranked among themselves; the ids of ranks below k, in
// list order, into chosen.  Returns the count, or -1 (nothing written) when
// more than 512 keys pass.  `hist` holds 16 + 16 * 8 + 2 * 8 ints.
__device__ int merge_bounded(const uint64_t *keys, const int *ids, int n, int k, int *scratch, int *chosen,
                             int *hist) {
    constexpr int NW = kLsaThreads / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned below = (1u << lane) - 1u;
    const int J = (n + kLsaThreads - 1) / kLsaThreads;
    uint64_t *wlow = reinterpret_cast<uint64_t *>(hist);      // [8]
    int *cnt = hist + 16;                                     // [16][8]
    int *rcnt = hist + 16 + 16 * NW;                          // [2][8]
    uint64_t tmax = 0ull;
    for (int j = 0; j < J; ++j) {
        const int i = j * kLsaThreads + tid;
        if (i < n) tmax = max(tmax, keys[i]);
    }
    const uint64_t lw = warp_kth_largest64(tmax, (k + NW - 1) / NW);
    if (lane == 0) wlow[warp] = lw;
    __syncthreads();
    uint64_t L = ~0ull;
#pragma unroll
    for (int w = 0; w < NW; ++w) L = min(L, wlow[w]);
    for (int j = 0; j < J; ++j) {
        const int i = j * kLsaThreads + tid;
        const unsigned bal = __ballot_sync(0xffffffffu, i < n && keys[i] >= L);
        if (lane == 0) cnt[j * NW + warp] = __popc(bal);
    }
    __syncthreads();
    int m = 0;
    for (int x = 0; x < J * NW; ++x) m += cnt[x];
    if (m > 512) {
        __syncthreads();          // every thread has read the counts before hist is reused
        return -1;
    }
    uint64_t *ckey = reinterpret_cast<uint64_t *>(scratch);  // [512]
    int *cid = scratch + 1024;                                // [512]
    int base = 0;
    for (int j = 0; j < J; ++j) {
        const int i = j * kLsaThreads + tid;
        const bool p = i < n && keys[i] >= L;
        const unsigned bal = __ballot_sync(0xffffffffu, p);
        int before = 0, tot = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const int c = cnt[j * NW + w];
            if (w < warp) before += c;
            tot += c;
        }
        if (p) {
            const int at = base + before + __popc(bal & below);
            ckey[at] = keys[i];
            cid[at] = ids[i];
        }
        base += tot;
    }
    __syncthreads();
    unsigned sb[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int c = rr * kLsaThreads + tid;
        bool sel = false;
        if (c < m) {
            const uint64_t x = ckey[c];
            int rk = 0;
            for (int jj = 0; jj < m; ++jj) {
                const uint64_t y = ckey[jj];
                rk += (y > x) | ((y == x) & (jj < c));
            }
            sel = rk < k;
        }
        sb[rr] = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) rcnt[rr * NW + warp] = __popc(sb[rr]);
    }
    __syncthreads();
    int ob = 0;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        int before = 0, tot = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const int c = rcnt[rr * NW + w];
            if (w < warp) before += c;
            tot += c;
        }
        if ((sb[rr] >> lane) & 1u) chosen[ob + before + __popc(sb[rr] & below)] = cid[rr * kLsaThreads + tid];
        ob += tot;
    }
    __syncthreads();
    return ob;
}

template <typename T>
__global__ void __launch_bounds__(kLsaThreads) lsa_select_kernel(LsaDecArgs a) {
    extern __shared__ __align__(16) unsigned char smraw[];
    const LsaShape &s = a.s;
    const LsaDecPlan &pl = a.pl;
    double *qbar = reinterpret_cast<double *>(smraw);                           // [d]
    int *red = reinterpret_cast<int *>(qbar + s.d);                             // [8]
    int *flag = red + 8;                                                        // [8]
    int *hist = flag + 8;                                                       // [264]
    uint64_t *keys = reinterpret_cast<uint64_t *>(hist + 264);                  // [max(CH, S*kk)]
    const int kmax = max(pl.CH, pl.S * pl.kk);
    int *ids = reinterpret_cast<int *>(keys + kmax);                            // [max(CH, S*kk)]
    int *pos = ids + kmax;                                                      // [max(CH, S*kk)]
    int *chosen = pos + kmax;                                                   // [ntop]
    int *off = chosen + pl.ntop;                                                // [ntop + 1]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bg = blockIdx.x / pl.S, chunk = blockIdx.x % pl.S;
    const int b = bg / s.Hkv, g = bg % s.Hkv;
    const int D = s.d;
    const T *q = (const T *)a.q;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the attention may start early
    for (int e = tid; e < D; e += kLsaThreads) {
        double acc = 0.0;
        for (int h = 0; h < s.G; ++h) acc += (double)to_f(q[((size_t)b * s.Hq + g * s.G + h) * D + e]);
        qbar[e] = acc / s.G;
    }
    __syncthreads();
    // scores of the chunk: a warp per centre, 16-byte loads, four centres in flight
    const int c0 = chunk * pl.CH, n = max(0, min(s.ctotal, c0 + pl.CH) - c0);
    const double *cb = a.centres + ((size_t)bg * s.ctotal + c0) * D;
    const int epl = D / 32;                    // doubles per lane: 2 (d 64) or 4 (d 128)
    double qv[4];                              // this lane's slice of the pooled query
#pragma unroll
    for (int e = 0; e < 4; ++e) qv[e] = e < epl ? qbar[lane * epl + e] : 0.0;
    bool nan_seen = false;
    for (int c = warp * 4; c < n; c += 4 * (kLsaThreads / 32)) {
        double part[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int cc = min(c + u, n - 1);
            const double *row = cb + (size_t)cc * D + lane * epl;
            double acc = 0.0;
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                if (e < epl) {
                    const double2 v = *reinterpret_cast<const double2 *>(row + e);
                    acc = fma(v.x, qv[e], acc);
                    acc = fma(v.y, qv[e + 1], acc);
                }
            }
            part[u] = acc;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part[u] += __shfl_xor_sync(0xffffffffu, part[u], o);
            if (lane == 0 && c + u < n) {
                const double sc = (double)s.scale * part[u];
                nan_seen |= isnan(sc);
                keys[c + u] = ord_key64(sc);
            }
        }
    }
    if (nan_seen) set_status(a.status, kStatusNaN);
    __syncthreads();
    if (pl.S == 1) {
        const int nsel = block_topk64(keys, n, pl.ntop, pos, hist, red);
        for (int i = tid; i < nsel; i += kLsaThreads) chosen[i] = c0 + pos[i];
        __syncthreads();
        expand_positions(a, bg, chosen, nsel, off, red);
        return;
    }
    // the chunk's candidates (ascending id) for the merge: every score, or its best kk
    int nsel = n;
    if (pl.kk < pl.CH) {
        nsel = block_topk64(keys, n, pl.kk, pos, hist, red);
    } else {
        for (int i = tid; i < n; i += kLsaThreads) pos[i] = i;
        __syncthreads();
    }
    uint64_t *pk = a.pkey + ((size_t)bg * pl.S + chunk) * pl.kk;
    int32_t *pi = a.pid + ((size_t)bg * pl.S + chunk) * pl.kk;
    for (int i = tid; i < nsel; i += kLsaThreads) {
        pk[i] = keys[pos[i]];
        pi[i] = c0 + pos[i];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) flag[0] = atomicAdd(a.done1 + bg, 1u) == (unsigned)(pl.S - 1);
    __syncthreads();
    if (!flag[0]) return;
    __threadfence();
    // merge: chunk c holds min(kk, its centres) candidates, packed in chunk order
    int ntot = 0;
    for (int c = 0; c < pl.S; ++c) ntot += min(pl.kk, max(0, min(s.ctotal, (c + 1) * pl.CH) - c * pl.CH));
    // (eight entries per thread loaded before any is stored: one round of loads)
    for (int e0 = 0; e0 < pl.S * pl.kk; e0 += 8 * kLsaThreads) {
        unsigned long long kv[8];
        int iv[8], dst[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = e0 + u * kLsaThreads + tid;
            dst[u] = -1;
            if (e < pl.S * pl.kk) {
                const int c = e / pl.kk, i = e % pl.kk;
                const int nv = min(pl.kk, max(0, min(s.ctotal, (c + 1) * pl.CH) - c * pl.CH));
                if (i < nv) {
                    // chunks before the last are full: c * min(kk, CH) candidates precede chunk c
                    dst[u] = c * min(pl.kk, pl.CH) + i;
                    const size_t src = ((size_t)bg * pl.S + c) * pl.kk + i;
                    kv[u] = __ldcg(reinterpret_cast<const unsigned long long *>(a.pkey) + src);
                    iv[u] = __ldcg(a.pid + src);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (dst[u] >= 0) {
                keys[dst[u]] = kv[u];
                ids[dst[u]] = iv[u];
            }
    }
    __syncthreads();
    // most lists: a bound, then a few hundred keys ranked; else the radix select
    int nfin = -1;
    if (ntot >= 1024 && ntot <= 16 * kLsaThreads && pl.ntop <= 256 && kmax >= 1536 &&
        (reinterpret_cast<uintptr_t>(pos) & 7u) == 0)
        nfin = merge_bounded(keys, ids, ntot, pl.ntop, pos, chosen, hist);
    if (nfin < 0) {
        nfin = block_topk64(keys, ntot, pl.ntop, pos, hist, red);
        for (int i = tid; i < nfin; i += kLsaThreads) chosen[i] = ids[pos[i]];
    }
    if (tid == 0) a.done1[bg] = 0u;
    __syncthreads();
    expand_positions(a, bg, chosen, nfin, off, red);
}

// Kernel 3 (flat decode, step 2): P CTAs per (batch, kv-head), each taking
// an equal share of the kept positions and walking it in rounds: a round's
// positions are staged in shared memory from the flat list, then a VPR-lane
// group per key row streams K and V with 16-byte loads (four rows per group
// in flight) and keeps an online softmax (fp32, exp2 domain) per query head of
// the pass.  Lane groups, warps and finally the CTAs of a (batch, kv-head) are
// merged by log-sum-exp; the last CTA writes o and lse.
template <typename T, int HG>
__global__ void __launch_bounds__(kLsaThreads, 2) lsa_attend_kernel(LsaDecArgs a) {
    constexpr float kLog2e = 1.4426950408889634f, kLn2 = 0.6931471805599453f;
    constexpr int EPV = 16 / (int)sizeof(T);
    extern __shared__ __align__(16) unsigned char smraw[];
    const LsaShape &s = a.s;
    const LsaDecPlan &pl = a.pl;
    const int D = s.d, VPR = D / EPV, RPW = 32 / VPR;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sub = lane / VPR, cv = lane % VPR;
    const int bg = blockIdx.x / pl.P, pi = blockIdx.x % pl.P;
    const int b = bg / s.Hkv, g = bg % s.Hkv;
    int *posv = reinterpret_cast<int *>(smraw);                                // [slice]
    float *wst = reinterpret_cast<float *>(posv + ((pl.slice + 3) & ~3));      // [8 warps][HG][D + 2]
    int *misc = reinterpret_cast<int *>(wst + max((kLsaThreads / 32) * HG * (D + 2), 2 * pl.P * s.G + 2 * s.G));   // [4]

    const int32_t *plist = a.pos + (size_t)bg * pl.pmax;
    const T *Kb = (const T *)a.K + (size_t)bg * s.N * D;
    const T *Vb = (const T *)a.V + (size_t)bg * s.N * D;
    const float sl2 = s.scale * kLog2e;
    // Every list is [sink][the chosen clusters' keys][window], in that order,
    // and the sink's and the window's rows are known before the list is: a CTA
    // first attends to its share of those (part 0), while the launch before
    // this one is still choosing the clusters, then to its share of the
    // clusters' keys (part 1, list entries sink_n .. tot - nfix).
    const int sink_n = min(s.sink, s.N), win0 = max(sink_n, s.N - s.window);
    const int nfix = sink_n + (s.N - win0);
    const int x0 = (int)((long long)nfix * pi / pl.P), x1 = (int)((long long)nfix * (pi + 1) / pl.P);
    int c0 = 0, c1 = 0;
    bool listed = false;
    for (int h0 = 0; h0 < s.G; h0 += HG) {
        const int nh = min(HG, s.G - h0);
        float qf[HG][EPV], acc[HG][EPV], m[HG], l[HG];
#pragma unroll
        for (int h = 0; h < HG; ++h) {
            if (h < nh) load16((const T *)a.q + ((size_t)b * s.Hq + g * s.G + h0 + h) * D + cv * EPV, qf[h]);
#pragma unroll
            for (int e = 0; e < EPV; ++e) {
                if (h >= nh) qf[h][e] = 0.f;
                qf[h][e] *= sl2;
                acc[h][e] = 0.f;
            }
            m[h] = -CUDART_INF_F;
            l[h] = 0.f;
        }
        for (int part = 0; part < 2; ++part) {
            if (part == 1 && !listed) {
                asm volatile("griddepcontrol.wait;" ::: "memory");   // the list comes from the launch before this one
                const int mid = max(0, min(a.cnt[2 * (size_t)bg + 1], pl.pmax) - nfix);
                c0 = sink_n + (int)((long long)mid * pi / pl.P);
                c1 = sink_n + (int)((long long)mid * (pi + 1) / pl.P);
                listed = true;
            }
            const int t0 = part == 0 ? x0 : c0, t1 = part == 0 ? x1 : c1;
            // the part's positions, walked in rounds of pl.slice
            for (int r0 = t0; r0 < t1; r0 += pl.slice) {
                const int r1 = min(t1, r0 + pl.slice);
                __syncthreads();                             // the previous round's positions are read
                for (int i = tid; i < r1 - r0; i += kLsaThreads) {
                    const int r = r0 + i;
                    posv[i] = part == 1 ? plist[r] : r < sink_n ? r : win0 + (r - sink_n);
                    SA_CHECK_START(a.status, posv[i], s.N);
                }
                __syncthreads();
                const int np = r1 - r0;
                // rows of this lane group: vb + sub + u * RPW * 8 for the warp's bases vb
                // (the trip count is the same for every lane: the row reductions
                // shuffle over the whole warp); two rows per group in flight
                constexpr int U = 4, NW = kLsaThreads / 32;
                for (int vb = warp * RPW; vb < np; vb += U * RPW * NW) {
                    uint4 kr[U], vr[U];
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int v = min(vb + sub + u * RPW * NW, np - 1);
                        const size_t row = (size_t)posv[v] * D + cv * EPV;
                        kr[u] = *reinterpret_cast<const uint4 *>(Kb + row);
                        vr[u] = *reinterpret_cast<const uint4 *>(Vb + row);
                    }
                    // the U rows' scores for every head of the pass (summed over the lane group)
                    float z[U][HG];
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        float kf[EPV];
                        load16(reinterpret_cast<const T *>(&kr[u]), kf);
#pragma unroll
                        for (int h = 0; h < HG; ++h) {
                            float t = 0.f;
#pragma unroll
                            for (int e = 0; e < EPV; ++e) t = fmaf(qf[h][e], kf[e], t);
                            for (int o = VPR / 2; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
                            // rows past the round (uniform over the lane group) and padded heads take no part
                            z[u][h] = (vb + sub + u * RPW * NW < np && h < nh) ? t : -CUDART_INF_F;
                        }
                    }
                    // one online-softmax step per head for the U rows: a single rescale
#pragma unroll
                    for (int h = 0; h < HG; ++h) {
                        float mn = m[h];
#pragma unroll
                        for (int u = 0; u < U; ++u) mn = fmaxf(mn, z[u][h]);
                        if (mn == -CUDART_INF_F) {
#pragma unroll
                            for (int u = 0; u < U; ++u) z[u][h] = 0.f;
                            continue;
                        }
                        const float corr = m[h] == -CUDART_INF_F ? 0.f : exp2f(m[h] - mn);
                        float ps = 0.f;
#pragma unroll
                        for (int u = 0; u < U; ++u) {
                            z[u][h] = exp2f(z[u][h] - mn);      // -inf rows give 0
                            ps += z[u][h];
                        }
                        l[h] = l[h] * corr + ps;
#pragma unroll
                        for (int e = 0; e < EPV; ++e) acc[h][e] *= corr;
                        m[h] = mn;
                    }
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        float vf[EPV];
                        load16(reinterpret_cast<const T *>(&vr[u]), vf);
#pragma unroll
                        for (int h = 0; h < HG; ++h)
#pragma unroll
                            for (int e = 0; e < EPV; ++e) acc[h][e] = fmaf(z[u][h], vf[e], acc[h][e]);
                    }
                }
            }
        }
        // merge the warp's lane groups (lanes VPR apart hold the same columns)
#pragma unroll
        for (int h = 0; h < HG; ++h) {
            for (int o = VPR; o < 32; o <<= 1) {
                const float mo = __shfl_xor_sync(0xffffffffu, m[h], o);
                const float lo = __shfl_xor_sync(0xffffffffu, l[h], o);
                const float mn = fmaxf(m[h], mo);
                const float f0 = m[h] == -CUDART_INF_F ? 0.f : exp2f(m[h] - mn);
                const float f1 = mo == -CUDART_INF_F ? 0.f : exp2f(mo - mn);
#pragma unroll
                for (int e = 0; e < EPV; ++e) {
                    const float ao = __shfl_xor_sync(0xffffffffu, acc[h][e], o);
                    acc[h][e] = acc[h][e] * f0 + ao * f1;
                }
                l[h] = l[h] * f0 + lo * f1;
                m[h] = mn;
            }
            if (sub == 0) {
                float *w = wst + (warp * HG + h) * (D + 2);
#pragma unroll
                for (int e = 0; e < EPV; ++e) w[2 + cv * EPV + e] = acc[h][e];
                if (cv == 0) {
                    w[0] = m[h];
                    w[1] = l[h];
                }
            }
        }
        __syncthreads();
        // merge the warps; this CTA's partial per head
        for (int x = tid; x < nh * (D + 2); x += kLsaThreads) {
            const int h = x / (D + 2), e = x % (D + 2);
            float M = -CUDART_INF_F;
            for (int w = 0; w < kLsaThreads / 32; ++w) M = fmaxf(M, wst[(w * HG + h) * (D + 2)]);
            float val = 0.f;
            if (e == 0) {
                val = M;
            } else {
                for (int w = 0; w < kLsaThreads / 32; ++w) {
                    const float *ww = wst + (w * HG + h) * (D + 2);
                    if (ww[0] != -CUDART_INF_F) val = fmaf(ww[e], exp2f(ww[0] - M), val);
                }
            }
            a.part[(((size_t)bg * pl.P + pi) * s.G + h0 + h) * (D + 2) + e] = val;
        }
        __syncthreads();
    }
    // the last CTA of this (batch, kv-head) merges the partials
    __threadfence();
    __syncthreads();
    if (tid == 0) misc[2] = atomicAdd(a.done2 + bg, 1u) == (unsigned)(pl.P - 1);
    __syncthreads();
    if (!misc[2]) return;
    __threadfence();
    // the P partials: (m, l) of each into shared memory, per head the max M and
    // the sum L, then each partial's weight 2^(m - M); the accumulators are then
    // read with independent loads
    const float *pb = a.part + (size_t)bg * pl.P * s.G * (D + 2);
    float *wm = wst, *wl = wm + pl.P * s.G, *Mh = wl + pl.P * s.G, *Lh = Mh + s.G;
    for (int i = tid; i < pl.P * s.G; i += kLsaThreads) {
        wm[i] = __ldcg(pb + (size_t)i * (D + 2));
        wl[i] = __ldcg(pb + (size_t)i * (D + 2) + 1);
    }
    __syncthreads();
    for (int h = tid; h < s.G; h += kLsaThreads) {
        float M = -CUDART_INF_F, L = 0.f;
        for (int p = 0; p < pl.P; ++p) M = fmaxf(M, wm[p * s.G + h]);
        if (M != -CUDART_INF_F)
            for (int p = 0; p < pl.P; ++p)
                if (wm[p * s.G + h] != -CUDART_INF_F) L = fmaf(wl[p * s.G + h], exp2f(wm[p * s.G + h] - M), L);
        Mh[h] = M;
        Lh[h] = L;
    }
    __syncthreads();
    for (int i = tid; i < pl.P * s.G; i += kLsaThreads) {
        const float M = Mh[i % s.G];
        wm[i] = (wm[i] == -CUDART_INF_F || M == -CUDART_INF_F) ? 0.f : exp2f(wm[i] - M);
    }
    __syncthreads();
    for (int x = tid; x < s.G * D; x += kLsaThreads) {
        const int h = x / D, e = x % D;
        float O = 0.f;
#pragma unroll 8
        for (int p = 0; p < pl.P; ++p) O = fmaf(__ldcg(pb + ((size_t)p * s.G + h) * (D + 2) + 2 + e), wm[p * s.G + h], O);
        const float M = Mh[h], L = Lh[h];
        const size_t oh = (size_t)b * s.Hq + g * s.G + h;
        from_f(((T *)a.o)[oh * D + e], L > 0.f ? O / L : 0.f);
        if (e == 0) a.lse[oh] = L > 0.f ? (M + log2f(L)) * kLn2 : -CUDART_INF_F;
    }
    if (tid == 0) a.done2[bg] = 0u;
}

}  // namespace

size_t lsa_build_smem(const LsaShape &s) {
    return sizeof(double) * ((size_t)s.seg * s.d + kLsaThreads) + sizeof(int) * (3 * (size_t)s.seg + kLsaThreads);
}

cudaError_t launch_lsa_build(const LsaShape &s, const void *K, double *centres, int32_t *members, int32_t *sizes,
                             cudaStream_t st) {
    if (s.nseg == 0) return cudaSuccess;
    const size_t smem = lsa_build_smem(s);
    void (*kern)(LsaShape, const void *, double *, int32_t *, int32_t *) =
        s.dtype == SA_BF16 ? lsa_build_kernel<__nv_bfloat16> : lsa_build_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(s.B * s.Hkv * s.nseg), kLsaThreads, smem, st>>>(s, K, centres, members, sizes);
    note_launch();
    return cudaGetLastError();
}

bool lsa_decode_plan(const LsaShape &s, LsaDecPlan &pl, bool chunks) {
    const int C = s.ctotal;
    const int top = s.top_clusters;
    pl.ntop = min(top, C);
    if (pl.ntop == 0 || !chunks) {
        // nothing to choose: one CTA per (batch, kv-head) lays out the sink and the window
        pl.CH = 0;
        pl.S = 1;
        pl.kk = 0;
    } else {
        // chunks of 128 centres or more, so that the grid is one wave (four
        // CTAs per SM); the merge takes every score when it can hold them all
        // (C <= 4096), else each chunk passes its best min(top, CH), the chunks
        // grown until the merge's candidates fit one CTA
        const long long bgs = (long long)s.B * s.Hkv;
        pl.CH = 128;
        while (pl.CH < 4096 && bgs * ((C + pl.CH - 1) / pl.CH) > 4 * 148) pl.CH *= 2;
        pl.S = max(1, (C + pl.CH - 1) / pl.CH);
        if (C <= 4096) {
            pl.kk = pl.CH;
        } else {
            while (pl.S > 1 && (long long)pl.S * min(top, pl.CH) > 12288 && pl.CH < 8192) {
                pl.CH *= 2;
                pl.S = max(1, (C + pl.CH - 1) / pl.CH);
            }
            pl.kk = min(top, pl.CH);
        }
    }
    if (pl.CH > 8192 || (pl.S > 1 && (long long)pl.S * pl.kk > 12288)) return false;
    const long long sink_n = min(s.sink, s.N);
    // what the expansion can write even for an index whose clusters share items
    const long long bound = sink_n + min((long long)s.window, (long long)s.N) + (long long)pl.ntop * s.seg * s.pool;
    if (bound > (1LL << 30)) return false;
    pl.pmax = (int)max(1LL, bound);
    const int bgs = s.B * s.Hkv;
    // one wave of the attention kernel (two CTAs per SM), but at least 32
    // positions per CTA at the bound
    long long P = min(64LL, max(1LL, 2LL * 148 / bgs));
    P = min(P, (bound + 31) / 32);
    pl.P = (int)max(1LL, P);
    pl.slice = 1024;
    pl.HG = s.G >= 4 ? 4 : s.G >= 2 ? 2 : 1;     // query heads per pass (more would cost occupancy)
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    size_t off = kStatusBytes;
    pl.off_key = off;   off += al((size_t)bgs * pl.S * max(1, pl.kk) * 8);
    pl.off_id = off;    off += al((size_t)bgs * pl.S * max(1, pl.kk) * 4);
    pl.off_done1 = off; off += al((size_t)bgs * 4);
    pl.off_pos = off;   off += al((size_t)bgs * pl.pmax * 4);
    pl.off_cnt = off;   off += al((size_t)bgs * 8);
    pl.off_part = off;  off += al((size_t)bgs * pl.P * s.G * (s.d + 2) * 4);
    pl.off_done2 = off; off += al((size_t)bgs * 4);
    pl.bytes = off;
    return true;
}

static size_t select_smem(const LsaShape &s, const LsaDecPlan &pl) {
    const size_t kmax = (size_t)max(pl.CH, pl.S * pl.kk);
    return sizeof(double) * s.d + (8 + 8 + 264) * 4 + kmax * (8 + 4 + 4) + (2 * (size_t)pl.ntop + 1) * 4;
}

static size_t attend_smem(const LsaShape &s, const LsaDecPlan &pl) {
    // the warps' states, or the last CTA's merge weights (2 P G + 2 G floats), whichever is larger
    const size_t wst = max((size_t)(kLsaThreads / 32) * pl.HG * (s.d + 2), 2 * (size_t)pl.P * s.G + 2 * (size_t)s.G);
    return (size_t)((pl.slice + 3) & ~3) * 4 + wst * 4 + 16;
}

template <typename T>
static cudaError_t run_lsa_attend(const LsaDecArgs &a, cudaStream_t st) {
    const LsaShape &s = a.s;
    const LsaDecPlan &pl = a.pl;
    void (*k2)(LsaDecArgs) = nullptr;
    switch (pl.HG) {
        case 1: k2 = lsa_attend_kernel<T, 1>; break;
        case 2: k2 = lsa_attend_kernel<T, 2>; break;
        default: k2 = lsa_attend_kernel<T, 4>; break;
    }
    const size_t sm2 = attend_smem(s, pl);
    cudaError_t e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    if (e != cudaSuccess) return e;
    e = launch_pdl(k2, dim3((unsigned)(s.B * s.Hkv) * pl.P), dim3(kLsaThreads), sm2, st, a);
    note_launch();
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_lsa_attend(const LsaDecArgs &a, cudaStream_t st) {
    return a.s.dtype == SA_BF16 ? run_lsa_attend<__nv_bfloat16>(a, st) : run_lsa_attend<float>(a, st);
}

void lsa_bind_workspace(LsaDecArgs &a, void *ws) {
    unsigned char *w = static_cast<unsigned char *>(ws);
    const LsaDecPlan &pl = a.pl;
    a.status = reinterpret_cast<unsigned *>(w);
    a.pkey = reinterpret_cast<uint64_t *>(w + pl.off_key);
    a.pid = reinterpret_cast<int32_t *>(w + pl.off_id);
    a.done1 = reinterpret_cast<unsigned *>(w + pl.off_done1);
    a.pos = reinterpret_cast<int32_t *>(w + pl.off_pos);
    a.cnt = reinterpret_cast<int32_t *>(w + pl.off_cnt);
    a.part = reinterpret_cast<float *>(w + pl.off_part);
    a.done2 = reinterpret_cast<unsigned *>(w + pl.off_done2);
}

template <typename T>
static cudaError_t run_lsa_select(const LsaDecArgs &a, cudaStream_t st) {
    const LsaShape &s = a.s;
    const LsaDecPlan &pl = a.pl;
    const size_t sm1 = select_smem(s, pl);
    cudaError_t e = cudaFuncSetAttribute(lsa_select_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
    if (e != cudaSuccess) return e;
    lsa_select_kernel<T><<<(unsigned)(s.B * s.Hkv) * pl.S, kLsaThreads, sm1, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_lsa_decode(const LsaShape &s, const LsaDecPlan &pl, const void *q, const void *K, const void *V,
                              const double *centres, const int32_t *members, const int32_t *sizes, void *ws,
                              void *o, float *lse, int32_t *kept, cudaStream_t st) {
    LsaDecArgs a{};
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
    cudaError_t e = s.dtype == SA_BF16 ? run_lsa_select<__nv_bfloat16>(a, st) : run_lsa_select<float>(a, st);
    if (e != cudaSuccess) return e;
    return launch_lsa_attend(a, st);
}

}  // namespace sa
