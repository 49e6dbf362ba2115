// lsa.cuh -- internal interface of the clustered index (lsa.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sa {

// Shape of one flat-index call, resolved on the host.
struct LsaShape {
    int B, Hq, Hkv, G, d, N, pool, seg, clusters, top_clusters, sink, window, dtype;
    float scale;
    int nseg;        // complete segments: N / (pool * seg)
    int ctotal;      // clusters per (batch, kv-head): nseg * clusters
};

// Work split and workspace layout of a decode through the index (host-side).
struct LsaDecPlan {
    int S;           // centre-score chunks per (batch, kv-head)
    int CH;          // centres per chunk
    int kk;          // candidates a chunk passes to the merge: CH when the merge holds every
                     // centre, else min(top_clusters, CH)
    int ntop;        // clusters chosen: min(top_clusters, ctotal)
    int pmax;        // kept key positions per (batch, kv-head), at most
    int P;           // attention CTAs per (batch, kv-head)
    int slice;       // key positions an attention CTA stages per round
    int HG;          // query heads per attention pass (1, 2 or 4)
    size_t off_key, off_id, off_done1, off_pos, off_cnt, off_part, off_done2, bytes;
};

struct LsaDecArgs {
    LsaShape s;
    LsaDecPlan pl;
    const void *q, *K, *V;
    const double *centres;
    const int32_t *members, *sizes;
    unsigned *status;
    uint64_t *pkey;       // [B*Hkv][S][kk] chunk candidates (keys)
    int32_t *pid;         // [B*Hkv][S][kk] chunk candidates (cluster ids)
    unsigned *done1;      // [B*Hkv] score chunks finished; back to 0 by the merging CTA
    int32_t *pos;         // [B*Hkv][pmax] kept key positions
    int32_t *cnt;         // [B*Hkv][2]: kept positions (twice)
    float *part;          // [B*Hkv][P][G][d + 2] attention partials (m, l, acc)
    unsigned *done2;      // [B*Hkv] attention CTAs finished; back to 0 by the merging CTA
    void *o;
    float *lse;
    int32_t *kept;        // optional [B*Hkv] kept positions
};

// false when the index is too large for the decode's single-CTA merge
// (`chunks` = false: a tree decode, which scans no chunks of centres)
bool lsa_decode_plan(const LsaShape &s, LsaDecPlan &pl, bool chunks = true);

// Tree over the flat index's clusters (lsa_tree.cu).
constexpr int kLsaMaxLevels = 24;
constexpr int kLsaTreeMaxLeaves = 4096;    // clusters per (batch, kv-head) a tree supports
struct LsaTreePlan {
    int L;                           // levels, the leaves (level 0) included
    int n[kLsaMaxLevels];            // nodes per level and (batch, kv-head)
    size_t off_mass[kLsaMaxLevels];  // every level: mass [B*Hkv][n] fp64 (key positions held)
    size_t off_cent[kLsaMaxLevels];  // level >= 1: centres [B*Hkv][n][d] fp64
    size_t off_cs[kLsaMaxLevels];    // level >= 1: first child [B*Hkv][n + 1]
    size_t off_ci[kLsaMaxLevels];    // level >= 1: children [B*Hkv][n of the level below], ascending per parent
    size_t bytes;                    // tree buffer
    size_t work_bytes;               // the build's working centres [B*Hkv][n0][d] fp64
    int maxfront;                    // most nodes a search level holds
};
bool lsa_tree_plan(const LsaShape &s, int fanout, LsaTreePlan &tp);
// `work`: the build's working centres, placed after every region a decode
// uses (the decode's completion counters must stay zero between calls)
cudaError_t launch_lsa_tree_build(const LsaShape &s, const LsaTreePlan &tp, const double *centres,
                                  const int32_t *sizes, void *tree, double *work, cudaStream_t st);
cudaError_t launch_lsa_tree_decode(const LsaShape &s, const LsaDecPlan &pl, const LsaTreePlan &tp, int beam,
                                   const void *q, const void *K, const void *V, const double *centres,
                                   const int32_t *members, const int32_t *sizes, const void *tree, void *ws, void *o,
                                   float *lse, int32_t *kept, int32_t *compared, cudaStream_t st);

cudaError_t launch_lsa_build(const LsaShape &s, const void *K, double *centres, int32_t *members, int32_t *sizes,
                             cudaStream_t st);
// Step 2 of a decode through the index: attention over the key positions that
// step 1 (flat scan or tree search) left in the workspace.
cudaError_t launch_lsa_attend(const LsaDecArgs &a, cudaStream_t st);
// Workspace pointers of a decode (layout of `pl`) filled into `a`.
void lsa_bind_workspace(LsaDecArgs &a, void *ws);
cudaError_t launch_lsa_decode(const LsaShape &s, const LsaDecPlan &pl, const void *q, const void *K, const void *V,
                              const double *centres, const int32_t *members, const int32_t *sizes, void *ws,
                              void *o, float *lse, int32_t *kept, cudaStream_t st);

}  // namespace sa
