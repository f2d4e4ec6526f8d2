// Small kernels that lay out the ranking problems of each entry point:
// row descriptors, PIVOT's groups and proxies, HISA's pooled keys and kept
// block lists.
#pragma once

#include "common.cuh"

namespace dsa {

// ------------------------------------------------------------------ dense
// One row per query: eligible keys s <= q_pos[t] of its sequence.
__global__ void dense_rows_kernel(const int32_t* q_off, const int32_t* k_off, const int32_t* q_pos,
                                  int32_t n_seqs, int32_t n_q, RowDesc* rows)
{
    grid_dep_launch();   // the unit builder may launch; it waits for these rows
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n_q) return;
    const int b = find_seq(q_off, n_seqs, t);
    rows[t] = RowDesc{t, b, eligible_count(q_pos[t], k_off[b + 1] - k_off[b]), 0};
}

// Dense top-k set-up in one launch, for a batch scored in one tensor-core launch (no row chunks):
// the workspace header cleared, one row per query (as dense_rows_kernel) and the launch's work
// units (as tc_units_kernel), each unit computed alone from the segments' tile offsets, which the
// host knows from the query offsets and passes in.  The units' key ranges come from the queries'
// positions directly, so the kernel does not wait on its own rows.
constexpr int kSetupMaxSeqs = 480;   // sequences whose tile offsets fit in the argument block

struct DenseSetupArgs {
    const int32_t* q_off;
    const int32_t* k_off;
    const int32_t* q_pos;
    RowDesc* rows;
    TcUnit* units;
    uint32_t* header;        // zeroed: header_words words
    int32_t header_words;
    int32_t n_seqs;
    int32_t n_q;
    int32_t TQ;              // query rows per tile
    int32_t splits;          // key-range parts per tile
    int32_t n_units;         // tile_base[n_seqs] * splits
    int32_t tile_base[kSetupMaxSeqs + 1];   // first tile of each sequence (tiles cut per sequence)
};

// Work unit u of a dense launch (u < a.n_units), computed alone; seq and L receive its sequence and
// that sequence's key count.
__device__ __forceinline__ TcUnit dense_unit(const DenseSetupArgs& a, int u, int& seq, int& L)
{
    const int tau = u / a.splits, s = u % a.splits;
    int lo = 0, hi = a.n_seqs - 1;   // the sequence whose tiles hold tile tau
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.tile_base[mid] <= tau) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int q0 = a.q_off[b], nq = a.q_off[b + 1] - q0;
    const int ntile = a.tile_base[b + 1] - a.tile_base[b];
    const int jj = ntile - 1 - (tau - a.tile_base[b]);   // longest causal tiles first
    const int r0 = q0 + jj * a.TQ;
    const int nr = min(a.TQ, nq - jj * a.TQ);
    const int kb = a.k_off[b];
    L = a.k_off[b + 1] - kb;
    seq = b;
    int maxnc = 0;
    for (int r = r0; r < r0 + nr; ++r) maxnc = max(maxnc, eligible_count(a.q_pos[r], L));
    const int nkt = (maxnc + 127) / 128;
    return TcUnit{r0, nr, nkt * s / a.splits, nkt * (s + 1) / a.splits, r0, kb, {0, 0}};
}

__global__ void dense_setup_kernel(const __grid_constant__ DenseSetupArgs a)
{
    grid_dep_launch();   // the scoring kernel may set up; it waits for this grid before reading units
    const int gid = blockIdx.x * blockDim.x + threadIdx.x;
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < a.header_words; i += blockDim.x) a.header[i] = 0u;
    if (gid < a.n_q) {
        const int b = find_seq(a.q_off, a.n_seqs, gid);
        a.rows[gid] = RowDesc{gid, b, eligible_count(a.q_pos[gid], a.k_off[b + 1] - a.k_off[b]), 0};
    }
    if (gid < a.n_units) {
        int seq, L;
        a.units[gid] = dense_unit(a, gid, seq, L);
    }
}

// Rows [r0, r0 + n) of a row array, with their query rows made relative to r0 (a row chunk whose
// queries sit in a buffer of their own).
__global__ void chunk_rows_kernel(const RowDesc* rows, int32_t r0, int32_t n, RowDesc* out)
{
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= n) return;
    RowDesc r = rows[r0 + j];
    r.qrow -= r0;
    out[j] = r;
}

// ------------------------------------------------------------------ PIVOT
// PIVOT ("PIVOT: Efficient Query-Group Indexing for Token-Level Sparse
// Attention", abstract): inside each sequence, consecutive runs of G query
// rows form a group; the group's proxy scans keys up to its last position.
struct GroupDesc {
    int32_t seq;
    int32_t first;    // first query row
    int32_t size;     // queries in the group (<= G)
    int32_t n_scan;   // keys the proxy scans: s < n_scan
};

// Single CTA: group_base[b] = number of groups before sequence b, then one
// GroupDesc and one proxy RowDesc per group.
__global__ void pivot_groups_kernel(const int32_t* q_off, const int32_t* k_off, const int32_t* q_pos,
                                    int32_t n_seqs, int32_t G, int32_t n_groups, int32_t* group_base,
                                    GroupDesc* groups, RowDesc* proxy_rows)
{
    if (threadIdx.x == 0) {
        int32_t acc = 0;
        for (int b = 0; b < n_seqs; ++b) {
            group_base[b] = acc;
            acc += (q_off[b + 1] - q_off[b] + G - 1) / G;
        }
        group_base[n_seqs] = acc;
    }
    __syncthreads();
    for (int g = threadIdx.x; g < n_groups; g += blockDim.x) {
        const int b = find_seq(group_base, n_seqs, g);
        const int first = q_off[b] + (g - group_base[b]) * G;
        const int size = min(G, q_off[b + 1] - first);
        int32_t p_last = -1;
        for (int j = 0; j < size; ++j) p_last = max(p_last, q_pos[first + j]);
        const int n_scan = eligible_count(p_last, k_off[b + 1] - k_off[b]);
        groups[g] = GroupDesc{b, first, size, n_scan};
        proxy_rows[g] = RowDesc{g, b, n_scan, g};
    }
}

// Nearest bf16 of a double, ties to even, from the format: 1 sign bit, 8
// exponent bits, 7 stored significand bits.  The double's 52-bit significand
// is cut after its top 7 bits and rounded on the 45 bits cut off; values
// below the smallest normal bf16 (2^-126) are rounded on the subnormal grid
// 2^-133.  Values stay far below the bf16 overflow threshold.
__device__ __forceinline__ uint16_t bf16_bits_rne(double x)
{
    const uint64_t u = (uint64_t)__double_as_longlong(x);
    const uint32_t sign = (uint32_t)(u >> 63) << 15;
    const int e = (int)((u >> 52) & 0x7ff) - 1023;
    if (x == 0.0) return (uint16_t)sign;
    if (e < -126) {
        const double m = fabs(x) * 0x1p133;           // exact power-of-two scaling
        const double r = rint(m);                       // ties to even
        return (uint16_t)(sign | (uint32_t)r);          // r == 128 encodes 2^-126
    }
    uint64_t mant = u & ((1ull << 52) - 1);
    uint64_t keep = mant >> 45;
    const uint64_t rest = mant & ((1ull << 45) - 1);
    const uint64_t half = 1ull << 44;
    uint32_t ex = (uint32_t)(e + 127);
    if (rest > half || (rest == half && (keep & 1))) {
        if (++keep == 128) { keep = 0; ++ex; }
    }
    return (uint16_t)(sign | (ex << 7) | (uint32_t)keep);
}

// One CTA per group: proxy q = bf16(mean of q) with the mean in double,
// proxy w = mean of w (double, stored fp32).
__global__ void pivot_proxy_kernel(const GroupDesc* groups, const __nv_bfloat16* Q, const float* W,
                                   int32_t H, int32_t D, __nv_bfloat16* Qp, float* Wp)
{
    const GroupDesc g = groups[blockIdx.x];
    const int HD8 = H * D / 8;   // 16-byte groups of 8 elements per query row (D >= 32)
    const uint4* q = reinterpret_cast<const uint4*>(Q);
    uint4* qp = reinterpret_cast<uint4*>(Qp) + (int64_t)blockIdx.x * HD8;
    for (int e8 = threadIdx.x; e8 < HD8; e8 += blockDim.x) {
        double s[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};   // summed in query order
        for (int j = 0; j < g.size; ++j) {
            const uint4 v = __ldg(q + (int64_t)(g.first + j) * HD8 + e8);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                s[2 * e] += (double)__uint_as_float(w[e] << 16);                 // low half: element 2e
                s[2 * e + 1] += (double)__uint_as_float(w[e] & 0xffff0000u);    // high half: element 2e+1
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            o[e] = (uint32_t)bf16_bits_rne(s[2 * e] / g.size) | ((uint32_t)bf16_bits_rne(s[2 * e + 1] / g.size) << 16);
        qp[e8] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        double s = 0.0;
        for (int j = 0; j < g.size; ++j) s += (double)W[(int64_t)(g.first + j) * H + h];
        Wp[(int64_t)blockIdx.x * H + h] = (float)(s / g.size);
    }
}

// One row per query for Reuse / Refine: the group's candidates (ascending,
// -1 padded) that lie inside the query's own prefix form a prefix of the
// candidate list; RowDesc.list = group.
// cand_len (nullable): usable length of each group's list (entries past it are ignored).
__global__ void pivot_query_rows_kernel(const int32_t* q_off, const int32_t* k_off, const int32_t* q_pos,
                                        int32_t n_seqs, int32_t n_q, int32_t G, const int32_t* group_base,
                                        const int32_t* cand, int32_t C, const int32_t* cand_len, RowDesc* rows)
{
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n_q) return;
    const int b = find_seq(q_off, n_seqs, t);
    const int g = group_base[b] + (t - q_off[b]) / G;
    const int lim = eligible_count(q_pos[t], k_off[b + 1] - k_off[b]);   // keys s < lim
    if (!cand) {   // no candidate list yet: the row's limit in key indices
        rows[t] = RowDesc{t, b, lim, g};
        return;
    }
    const int32_t* c = cand + (int64_t)g * C;
    int lo = 0, hi = cand_len ? cand_len[g] : C;   // first position whose candidate is >= lim or -1
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int32_t s = c[mid];
        if (s >= 0 && s < lim) lo = mid + 1; else hi = mid;
    }
    rows[t] = RowDesc{t, b, lo, g};
}

// Checks caller-supplied candidate lists (one warp per group): strictly ascending key indices of
// the group's sequence, then -1 padding.  len[g] = the usable prefix (up to the first -1 or the
// first bad entry); a bad entry records kErrBadRow with detail g.
__global__ void pivot_check_cand_kernel(const int32_t* cand, int32_t C, const GroupDesc* groups, int32_t n_groups,
                                        const int32_t* k_off, int32_t* len, uint32_t* status)
{
    const int g = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (g >= n_groups) return;
    const int seq = groups[g].seq;
    const int L = k_off[seq + 1] - k_off[seq];
    const int32_t* c = cand + (int64_t)g * C;
    int first_end = C, first_bad = C;
    for (int i = lane; i < C; i += 32) {
        const int32_t v = c[i];
        const int32_t prev = i > 0 ? c[i - 1] : -1;
        if (v < 0) { first_end = min(first_end, i); continue; }
        // a key outside the sequence, not above its predecessor, or after the padding
        if (v >= L || (i > 0 && (prev < 0 || prev >= v))) first_bad = min(first_bad, i);
    }
    first_end = __reduce_min_sync(0xffffffffu, first_end);
    first_bad = __reduce_min_sync(0xffffffffu, first_bad);
    if (lane == 0) {
        if (first_bad < C) record_error(status, kErrBadRow, (uint32_t)g);
        len[g] = min(first_end, first_bad);
    }
}

// ------------------------------------------------------------------- HISA
// HISA ("HISA: Efficient Hierarchical Indexing for Fine-Grained Sparse
// Attention", abstract): pooled block keys, block filter, token refinement.

// Pooled key of block j: mean of its keys (fp32 sum in token order).  One
// CTA of D threads per block; thread i owns dimension i (coalesced rows).
// The owning sequence is found by walking the key offsets (few sequences).
__global__ void hisa_pool_kernel(const __nv_bfloat16* K, const int32_t* k_off, int32_t n_seqs, int32_t B,
                                 int32_t D, float* pooled)
{
    __shared__ int32_t s_seq, s_first;
    const int j = blockIdx.x;
    if (threadIdx.x == 0) {
        int32_t acc = 0, b = 0;
        for (; b < n_seqs; ++b) {
            const int32_t nb = (k_off[b + 1] - k_off[b] + B - 1) / B;
            if (j < acc + nb) break;
            acc += nb;
        }
        s_seq = b;
        s_first = acc;
    }
    __syncthreads();
    const int b = s_seq;
    const int s0 = (j - s_first) * B;
    const int L = k_off[b + 1] - k_off[b];
    const int s1 = min(s0 + B, L);
    const uint16_t* k = reinterpret_cast<const uint16_t*>(K) + (int64_t)k_off[b] * D;
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
        float s = 0.f;
        for (int t = s0; t < s1; ++t) s += __uint_as_float((uint32_t)k[(int64_t)t * D + i] << 16);
        pooled[(int64_t)j * D + i] = s / (float)(s1 - s0);
    }
}

// HISA set-up in one launch: every CTA writes the block-scoring rows (the
// middle blocks 1 .. last-1 of query t; column c is block c + 1) and the
// per-query segment offsets query_off[t] = t of its queries; CTA 0 also
// writes block_base (first pooled block of each sequence) and clears the
// workspace header.
__global__ void hisa_setup_kernel(const int32_t* q_off, const int32_t* k_off, const int32_t* q_pos, int32_t n_seqs,
                                  int32_t n_q, int32_t B, int32_t* block_base, RowDesc* rows, int32_t* query_off,
                                  uint32_t* header, int32_t header_words)
{
    if (blockIdx.x == 0)   // the workspace header (status word, select counters) starts the call at zero
        for (int i = threadIdx.x; i < header_words; i += blockDim.x) header[i] = 0u;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        int32_t acc = 0;
        for (int b = 0; b < n_seqs; ++b) {
            block_base[b] = acc;
            acc += (k_off[b + 1] - k_off[b] + B - 1) / B;
        }
        block_base[n_seqs] = acc;
    }
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t > n_q) return;
    query_off[t] = t;
    if (t == n_q) return;
    const int b = find_seq(q_off, n_seqs, t);
    const int n = eligible_count(q_pos[t], k_off[b + 1] - k_off[b]);
    const int last = n > 0 ? (n - 1) / B : 0;
    rows[t] = RowDesc{t, b, last > 1 ? last - 1 : 0, t};
}

// The three bf16 planes of an fp32 value: v = hi + mid + lo exactly.  hi is v with its low 16
// mantissa bits cleared; the remainder v - hi (exact: at most 16 significant bits) is split the
// same way, and what is left after that has at most 8 significant bits, so it is a bf16 itself.
__device__ __forceinline__ void split_bf16x3(float v, uint32_t& hi, uint32_t& mid, uint32_t& lo)
{
    const uint32_t hb = __float_as_uint(v) & 0xffff0000u;
    const float r1 = v - __uint_as_float(hb);
    const uint32_t mb = __float_as_uint(r1) & 0xffff0000u;
    const float r2 = r1 - __uint_as_float(mb);
    hi = hb >> 16;
    mid = mb >> 16;
    lo = __float_as_uint(r2) >> 16;
}

// HISA's set-up for a block stage on the tensor cores, one launch.  CTAs [0, row_ctas): the
// workspace header cleared, query_off = 0..n_q, one block row per query (its middle blocks
// 1 .. last - 1 as columns 0 .. last - 2) and the block-scoring work units (as dense_setup_kernel's:
// tiles of TQ queries of one sequence, each tile's middle-block columns split `splits` ways; the key
// row of column 0 is the sequence's block 1 in plane 0).  The other CTAs split the pooled fp32 keys
// into the three bf16 planes the scoring kernel reads (plane p at rows p * n_blocks).
struct HisaSetupArgs {
    const int32_t* q_off;
    const int32_t* k_off;
    const int32_t* q_pos;
    const float* pooled;        // [n_blocks, D]
    uint32_t* planes;           // [3, n_blocks, D] bf16, as pairs
    RowDesc* rows;
    TcUnit* units;
    int32_t* query_off;
    uint32_t* header;           // zeroed: header_words words
    int64_t n_pairs;            // n_blocks * D / 2
    int32_t header_words;
    int32_t n_seqs;
    int32_t n_q;
    int32_t B;
    int32_t TQ;
    int32_t splits;
    int32_t n_units;
    int32_t row_ctas;
    int32_t tile_base[kSetupMaxSeqs + 1];    // first tile of each sequence
    int32_t block_base[kSetupMaxSeqs + 1];   // first pooled block of each sequence
};

__device__ __forceinline__ int32_t hisa_mid_count(int32_t pos, int32_t L, int32_t B)
{
    const int n = eligible_count(pos, L);
    const int last = n > 0 ? (n - 1) / B : 0;
    return last > 1 ? last - 1 : 0;
}

__global__ void hisa_setup_tc_kernel(const __grid_constant__ HisaSetupArgs a)
{
    grid_dep_launch();   // the scoring kernel may set up; it waits for this grid before reading units
    if ((int)blockIdx.x >= a.row_ctas) {
        const int64_t stride = (int64_t)(gridDim.x - a.row_ctas) * blockDim.x;
        const int64_t plane = a.n_pairs;   // 32-bit words per plane
        const float2* src = reinterpret_cast<const float2*>(a.pooled);
        for (int64_t i = (int64_t)(blockIdx.x - a.row_ctas) * blockDim.x + threadIdx.x; i < a.n_pairs; i += stride) {
            const float2 v = __ldg(src + i);
            uint32_t h0, m0, l0, h1, m1, l1;
            split_bf16x3(v.x, h0, m0, l0);
            split_bf16x3(v.y, h1, m1, l1);
            a.planes[i] = h0 | (h1 << 16);
            a.planes[plane + i] = m0 | (m1 << 16);
            a.planes[2 * plane + i] = l0 | (l1 << 16);
        }
        return;
    }
    const int gid = blockIdx.x * blockDim.x + threadIdx.x;
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < a.header_words; i += blockDim.x) a.header[i] = 0u;
    if (gid <= a.n_q) a.query_off[gid] = gid;
    if (gid < a.n_q) {
        const int b = find_seq(a.q_off, a.n_seqs, gid);
        a.rows[gid] = RowDesc{gid, b, hisa_mid_count(a.q_pos[gid], a.k_off[b + 1] - a.k_off[b], a.B), gid};
    }
    if (gid < a.n_units) {
        const int tau = gid / a.splits, s = gid % a.splits;
        int lo = 0, hi = a.n_seqs - 1;   // the sequence whose tiles hold tile tau
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (a.tile_base[mid] <= tau) lo = mid; else hi = mid - 1;
        }
        const int b = lo;
        const int q0 = a.q_off[b], nq = a.q_off[b + 1] - q0;
        const int jj = tau - a.tile_base[b];
        const int r0 = q0 + jj * a.TQ;
        const int nr = min(a.TQ, nq - jj * a.TQ);
        const int L = a.k_off[b + 1] - a.k_off[b];
        int maxnc = 0;
        for (int r = r0; r < r0 + nr; ++r) maxnc = max(maxnc, hisa_mid_count(a.q_pos[r], L, a.B));
        const int nkt = (maxnc + 127) / 128;
        a.units[gid] = TcUnit{r0, nr, nkt * s / a.splits, nkt * (s + 1) / a.splits, r0, a.block_base[b] + 1, {0, 0}};
    }
}

// Kept blocks of query t: block 0, the selected middle blocks (ascending,
// -1 padded), and the query's own block; then the token row over them.
__global__ void hisa_kept_kernel(const RowDesc* block_rows, const int32_t* mid, int32_t keep,
                                 const int32_t* q_pos, const int32_t* k_off, int32_t n_q, int32_t B,
                                 int32_t* kept, RowDesc* token_rows)
{
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n_q) return;
    const RowDesc br = block_rows[t];
    const int n = eligible_count(q_pos[t], k_off[br.seq + 1] - k_off[br.seq]);
    int32_t* out = kept + (int64_t)t * (keep + 2);
    int m = 0;
    int ncols = 0;
    if (n > 0) {
        const int last = (n - 1) / B;
        out[m++] = 0;
        for (int j = 0; j < keep; ++j) {
            const int32_t v = mid[(int64_t)t * keep + j];
            if (v < 0) break;
            out[m++] = v;
        }
        if (last > 0) out[m++] = last;
        ncols = (m - 1) * B + (n - last * B);
    }
    for (int j = m; j < keep + 2; ++j) out[j] = -1;
    token_rows[t] = RowDesc{t, br.seq, ncols, t};
}

// Kept blocks and token rows (as hisa_kept_kernel) and the token-scoring work units, one warp per
// query: the lanes read the query's selected middle blocks together (ascending, then -1), and the
// query's `splits` units cover the kept blocks' key tiles (a query is a segment of one row).
__global__ void hisa_kept_units_kernel(const RowDesc* block_rows, const int32_t* mid, int32_t keep,
                                       const int32_t* q_pos, const int32_t* k_off, int32_t n_q, int32_t B,
                                       int32_t splits, int32_t* kept, RowDesc* token_rows, TcUnit* units)
{
    grid_dep_wait();     // the block selection comes from the previous kernel
    grid_dep_launch();
    const int t = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    if (t >= n_q) return;   // (uniform per warp)
    const RowDesc br = block_rows[t];
    const int L = k_off[br.seq + 1] - k_off[br.seq];
    const int n = eligible_count(q_pos[t], L);
    const int last = n > 0 ? (n - 1) / B : 0;
    int32_t* out = kept + (int64_t)t * (keep + 2);
    // the selected middle blocks are packed first: count them a warp's width at a time
    int n_mid = 0;
    for (int j0 = 0; j0 < keep; j0 += 32) {
        const int j = j0 + lane;
        const int32_t v = j < keep ? mid[(int64_t)t * keep + j] : -1;
        if (v >= 0 && n > 0) out[1 + j] = v;
        n_mid += __popc(__ballot_sync(0xffffffffu, v >= 0));
    }
    if (n == 0) n_mid = 0;
    const int m = n > 0 ? 1 + n_mid + (last > 0 ? 1 : 0) : 0;   // kept blocks
    if (lane == 0 && n > 0) {
        out[0] = 0;
        if (last > 0) out[1 + n_mid] = last;
    }
    for (int j = m + lane; j < keep + 2; j += 32) out[j] = -1;
    const int ncols = m > 0 ? (m - 1) * B + (n - last * B) : 0;
    if (lane == 0) token_rows[t] = RowDesc{t, br.seq, ncols, t};
    const int nkt = (ncols + 127) / 128;
    for (int s = lane; s < splits; s += 32)
        units[(int64_t)t * splits + s] = TcUnit{t, 1, nkt * s / splits, nkt * (s + 1) / splits, t, k_off[br.seq], {0, 0}};
}

// ------------------------------------------------------ tensor-core units
// Work units of one tensor-core scoring launch over launch rows
// [0, n_rows) = absolute rows [row_base, row_base + n_rows).  Rows are cut into
// tiles of at most TQ consecutive rows of one segment (seg_off: absolute row
// offsets per segment); each tile's key tiles are split `splits` ways.
// Within a segment tiles are emitted last-first, so the longest causal tiles
// start first.  One CTA of 1024 threads; tile_base is [n_seg + 1] scratch.
__global__ void tc_units_kernel(const RowDesc* rows, int32_t n_rows, int32_t row_base, const int32_t* seg_off,
                                int32_t n_seg, int32_t TQ, int32_t splits, const int32_t* k_base, int32_t* tile_base,
                                TcUnit* units)
{
    __shared__ int32_t part[1024];
    grid_dep_wait();     // rows come from the previous kernel
    grid_dep_launch();   // the scoring kernel may set up while this runs
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (n_seg + nt - 1) / nt;   // contiguous segments per thread
    const int s0 = min(n_seg, tid * per), s1 = min(n_seg, s0 + per);
    auto tiles_of = [&](int b) {
        const int lo = max(seg_off[b], row_base), hi = min(seg_off[b + 1], row_base + n_rows);
        return hi > lo ? (hi - lo + TQ - 1) / TQ : 0;
    };
    int sum = 0;
    for (int b = s0; b < s1; ++b) sum += tiles_of(b);
    part[tid] = sum;
    __syncthreads();
    for (int o = 1; o < nt; o <<= 1) {   // inclusive scan of the per-thread sums
        const int x = tid >= o ? part[tid - o] : 0;
        __syncthreads();
        part[tid] += x;
        __syncthreads();
    }
    int acc = part[tid] - sum;
    for (int b = s0; b < s1; ++b) {
        tile_base[b] = acc;
        acc += tiles_of(b);
    }
    if (tid == nt - 1) tile_base[n_seg] = part[nt - 1];
    __syncthreads();
    const int total = tile_base[n_seg];
    for (int tau = tid; tau < total; tau += nt) {
        const int b = find_seq(tile_base, n_seg, tau);
        const int lo = max(seg_off[b], row_base), hi = min(seg_off[b + 1], row_base + n_rows);
        const int ntile = (hi - lo + TQ - 1) / TQ;
        const int jj = ntile - 1 - (tau - tile_base[b]);
        const int r0 = lo + jj * TQ - row_base;
        const int nr = min(TQ, hi - lo - jj * TQ);
        int maxnc = 0;
        for (int r = r0; r < r0 + nr; ++r) maxnc = max(maxnc, rows[r].ncols);
        const int nkt = (maxnc + 127) / 128;
        const RowDesc f = rows[r0];
        const int krow0 = k_base[f.seq];
        for (int s = 0; s < splits; ++s)
            units[tau * splits + s] = TcUnit{r0, nr, nkt * s / splits, nkt * (s + 1) / splits, f.qrow, krow0, {0, 0}};
    }
}

// Row offsets of PIVOT groups (segment g = rows [off[g], off[g+1])), for the
// tensor-core unit builder.
__global__ void group_row_offsets_kernel(const GroupDesc* groups, int32_t n_groups, int32_t n_q, int32_t* off)
{
    const int g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g < n_groups) off[g] = groups[g].first;
    if (g == 0) off[n_groups] = n_q;
}


// Fills a row-major [rows, cols] fp32 matrix with -inf (masked scores).
__global__ void fill_neg_inf_kernel(float* S, int64_t ld, int32_t rows, int32_t cols)
{
    const int64_t total = (int64_t)rows * cols;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x)
        S[(i / cols) * ld + (i % cols)] = -INFINITY;
}

}  // namespace dsa
