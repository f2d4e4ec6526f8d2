// PIVOT Reuse from one selection per group ("PIVOT: Efficient Query-Group
// Indexing for Token-Level Sparse Attention", abstract: the group shares the
// proxy's ranking; each query keeps the best of the candidates inside its own
// causal prefix).
//
// Every query of group g ranks the same candidate row (the proxy scores of
// the group's candidates, ascending key order) by (score desc, index asc);
// query t sees only its first ncols_t candidates.  Let L be the group's top
// kp = k + G - 1 candidates.  L restricted to a query's prefix is a prefix of
// that query's own ranking, so when it still holds >= k entries (always when
// at most G - 1 of L's entries lie past the query's position, as with
// consecutive positions) the query's top k is L restricted to its prefix
// minus its lowest-ranked surplus, and that surplus lies among L's kp - k
// lowest-ranked entries (the "tail").  Queries this does not cover (L holds
// too few of their candidates) are listed for the per-query selection.
#pragma once

#include "select.cuh"
#include "setup.cuh"

namespace dsa {

// One row per group over its candidate list: ncols = the candidates the proxy kept.
__global__ void pivot_cand_rows_kernel(const GroupDesc* groups, int32_t n_groups, int32_t C, RowDesc* rows)
{
    const int g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= n_groups) return;
    const GroupDesc gd = groups[g];
    rows[g] = RowDesc{g, gd.seq, min(C, gd.n_scan), g};
}

struct ReuseArgs {
    const GroupDesc* groups;
    const RowDesc* query_rows;   // ncols: the query's eligible candidates (a prefix of the group's list)
    const RowDesc* cand_rows;    // per group: ncols = candidates the proxy kept
    const int32_t* gsel;         // [n_groups, kp]: the group's top-kp candidate columns, ascending, -1 padded
    const float* gscore;         // [n_groups, kp]: their proxy scores
    int32_t kp;
    int32_t k;
    const int32_t* cand;         // [n_groups, C] candidate key indices, ascending; NULL: the group's list was
                                 // selected from the proxy row itself, so gsel holds key indices (a query's
                                 // row then has ncols = its key limit) and no candidate list exists yet
    int32_t C;
    int32_t n_groups;
    int32_t* gate;               // (cand NULL) set to n_groups when some query is left to the per-query selection
    int32_t* idx;                // [n_q, ld_idx]
    int64_t ld_idx;
    RowDesc* fb_rows;            // queries left to the per-query selection
    int32_t* fb_count;
    uint32_t* status;            // the workspace status word (checked builds record index errors there)
};

constexpr int kReuseThreads = 256;
constexpr int kReuseMaxTail = 64;   // kp - k = G - 1 <= 63

// Dynamic shared memory: columns and keys of the group's list.
__host__ __device__ inline size_t reuse_smem_bytes(int kp) { return (size_t)kp * 8; }

__global__ void __launch_bounds__(kReuseThreads) pivot_reuse_kernel(ReuseArgs a)
{
    constexpr int NT = kReuseThreads;
    extern __shared__ __align__(16) uint8_t reuse_smem[];
    int32_t* col = reinterpret_cast<int32_t*>(reuse_smem);
    uint32_t* key = reinterpret_cast<uint32_t*>(reuse_smem + (size_t)a.kp * 4);
    __shared__ SelScalars<NT> sh;
    __shared__ int32_t tail[kReuseMaxTail];      // list positions of the tail, collected in any order
    __shared__ int32_t tail_rk[kReuseMaxTail];   // the tail by rank, lowest first
    __shared__ int32_t drop_rk[kReuseMaxTail];   // one query's dropped list positions, rank order
    __shared__ int32_t drop_pos[kReuseMaxTail];  // the same, ascending
    __shared__ uint32_t s_tail_n;
    __shared__ int32_t s_m, s_drop, s_serve;

    const int g = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const GroupDesc gd = a.groups[g];
    const int ncols_g = a.cand_rows[g].ncols;
    const int n_list = min(ncols_g, a.kp);   // what the group selection returned
    const int k = a.k;
    for (int i = tid; i < n_list; i += NT) {
        col[i] = a.gsel[(int64_t)g * a.kp + i];
        key[i] = score_key(a.gscore[(int64_t)g * a.kp + i]);
    }
    if (tid == 0) s_tail_n = 0;
    const int n_tail = max(0, n_list - k);   // <= kp - k
    __syncthreads();

    if (n_tail > 0) {
        // ---- the tail: list entries below the k-th (ties at T past the first krem, in list order)
        int krem = k;
        const uint32_t T = radix_select<NT>([&](int i) { return key[i]; }, n_list, krem, sh.hist, sh.scratch);
        // tie ranks in list order: thread-contiguous runs, one block scan
        const int per = (n_list + NT - 1) / NT;
        const int i0 = min(n_list, tid * per), i1 = min(n_list, i0 + per);
        uint32_t ties = 0;
        for (int i = i0; i < i1; ++i) ties += key[i] == T;
        uint32_t incl = ties;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += x;
        }
        __syncthreads();   // radix_select's scratch and hist are free again
        if (lane == 31) sh.hist[warp] = incl;
        __syncthreads();
        uint32_t before = incl - ties;
        for (int w = 0; w < warp; ++w) before += sh.hist[w];
        for (int i = i0; i < i1; ++i) {
            const bool is_tie = key[i] == T;
            if (key[i] < T || (is_tie && before >= (uint32_t)krem)) {
                const uint32_t e = atomicAdd(&s_tail_n, 1u);
                if (DSA_CHECK(e < (uint32_t)kReuseMaxTail, a.status, 401)) tail[e] = i;   // the tail holds <= kp - k
            }
            before += is_tie;
        }
        __syncthreads();
        // ---- order the tail lowest rank first: smaller key, or equal key and later in the list
        if (warp == 0) {
            for (int e = lane; e < n_tail; e += 32) {
                const int pe = tail[e];
                int pos = 0;
                for (int f = 0; f < n_tail; ++f) {
                    const int pf = tail[f];
                    pos += key[pf] < key[pe] || (key[pf] == key[pe] && pf > pe);
                }
                tail_rk[pos] = pe;
            }
        }
        __syncthreads();
    }

    // ---- every query of the group
    for (int j = 0; j < gd.size; ++j) {
        const int t = gd.first + j;
        if (warp == 0) {
            const RowDesc rd = a.query_rows[t];
            const int nc = rd.ncols;
            int lo = 0, hi = n_list;   // m: list entries whose column is < nc
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (col[mid] < nc) lo = mid + 1; else hi = mid;
            }
            const int m = lo;
            const bool serve = m >= k || ncols_g <= a.kp;
            const int drop = serve ? max(0, m - k) : 0;
            // dropped: the `drop` lowest-ranked tail entries inside the prefix (position < m),
            // gathered in rank order, then put in list order
            uint32_t rank_base = 0;
            for (int e0 = 0; e0 < n_tail; e0 += 32) {
                const int e = e0 + lane;
                const int p = e < n_tail ? tail_rk[e] : 0;
                const bool in = e < n_tail && p < m;
                const uint32_t b = __ballot_sync(0xffffffffu, in);
                const uint32_t r = rank_base + __popc(b & lanemask_lt());
                if (in && r < (uint32_t)drop) drop_rk[r] = p;
                rank_base += __popc(b);
            }
            __syncwarp();
            for (int e = lane; e < drop; e += 32) {
                const int p = drop_rk[e];
                int order = 0;
                for (int f = 0; f < drop; ++f) order += drop_rk[f] < p;
                drop_pos[order] = p;
            }
            if (lane == 0) {
                s_m = m;
                s_drop = drop;
                s_serve = serve ? 1 : 0;
                if (!serve) {
                    a.fb_rows[atomicAdd(a.fb_count, 1)] = rd;
                    if (a.gate) *a.gate = a.n_groups;   // the candidate lists are needed after all
                }
            }
        }
        __syncthreads();
        if (s_serve) {
            const int m = s_m, drop = s_drop;
            int32_t* o = a.idx + (int64_t)t * a.ld_idx;
            const int32_t* cl = a.cand ? a.cand + (int64_t)g * a.C : nullptr;
            for (int i = tid; i < m; i += NT) {
                int lo = 0, hi = drop;   // dropped positions before i
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (drop_pos[mid] < i) lo = mid + 1; else hi = mid;
                }
                if (lo < drop && drop_pos[lo] == i) continue;
                if (!DSA_CHECK(i - lo < k && col[i] >= 0 && (!a.cand || col[i] < a.C), a.status, 402)) continue;
                o[i - lo] = a.cand ? cl[col[i]] : col[i];
            }
            for (int i = m - drop + tid; i < k; i += NT) o[i] = -1;
        }
        __syncthreads();
    }
}

// Reuse without a requested candidate list: the queries left to the per-query selection were listed
// with their key limit as ncols; once the candidate lists exist (a top-C selection gated on those
// queries), ncols becomes the count of the group's candidates below that limit.
__global__ void reuse_fallback_rows_kernel(RowDesc* fb_rows, const int32_t* fb_count, const int32_t* cand, int32_t C)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= *fb_count) return;
    RowDesc r = fb_rows[i];
    const int32_t* c = cand + (int64_t)r.list * C;
    int lo = 0, hi = C;   // first position whose candidate is >= the limit or -1
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int32_t s = c[mid];
        if (s >= 0 && s < r.ncols) lo = mid + 1; else hi = mid;
    }
    r.ncols = lo;
    fb_rows[i] = r;
}

}  // namespace dsa
