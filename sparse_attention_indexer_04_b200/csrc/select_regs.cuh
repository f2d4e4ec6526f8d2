// Exact per-row top-k of short rows held in registers: one CTA per row of at most NT * R columns,
// thread t holding the R consecutive columns [t R, t R + R).  For few short rows (HISA's block and
// token stages) the streaming select's sample, candidate pass and bitmaps are latency on the
// critical path; here the row is read once, the k-th largest key T is found by 8-bit radix passes
// over the registers (digits of key - min from the highest differing bit, stopping early when the
// rank's bin is taken whole: the same rule as radix_select_in), and one block-wide scan of the
// threads' (> T, == T) counts gives every selected column its output slot in column order, the
// ties at T going to the lowest columns.  The result is the streaming select's exactly.
#pragma once

#include "select.cuh"

namespace dsa {

// This thread's columns [c0, c0 + nv) of the row as keys (columns past n are not loaded).
template <int R>
__device__ __forceinline__ void regs_load(const float* src, int n, uint32_t (&key)[R], int& c0, int& nv)
{
    static_assert(R % 4 == 0, "16-byte loads");
    c0 = threadIdx.x * R;
    nv = max(0, min(R, n - c0));
    const float* p = src + c0;
    if (nv == R && (reinterpret_cast<uintptr_t>(p) & 15) == 0) {
#pragma unroll
        for (int j = 0; j < R; j += 4) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(p + j));
            key[j] = score_key(v.x); key[j + 1] = score_key(v.y);
            key[j + 2] = score_key(v.z); key[j + 3] = score_key(v.w);
        }
    } else {
#pragma unroll
        for (int j = 0; j < R; ++j) key[j] = j < nv ? score_key(__ldg(p + j)) : 0u;
    }
}

// The key T at rank krem (1 = largest) among every thread's first nv keys, and in krem the ties at
// T that rank reaches (0 when the passes stopped at a bin taken whole: then T is one below its
// lower edge).  All threads call it.
template <int NT, int R>
__device__ __forceinline__ uint32_t regs_radix(const uint32_t (&key)[R], int nv, int& krem, SelScalars<NT>& sh)
{
    constexpr int W = NT / 32;
    uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
    for (int j = 0; j < R; ++j)
        if (j < nv) { lo = min(lo, key[j]); hi = max(hi, key[j]); }
    block_key_range<NT>(lo, hi, sh.scratch);
    int top = 32 - __clz(hi - lo);   // bits of (key - lo) still undecided
    uint32_t prefix = 0;             // decided high bits of (T - lo)
    while (top > 0) {
        const int shift = max(top - 8, 0), width = top - shift;
        const uint32_t mask = (1u << width) - 1u;
        __syncthreads();
        for (int i = threadIdx.x; i < 256; i += NT) sh.hist[i] = 0;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < R; ++j) {
            const uint32_t rel = key[j] - lo;
            if (j < nv && ((rel >> 1) >> (top - 1)) == prefix) atomicAdd(&sh.hist[(rel >> shift) & mask], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) radix_pick(sh.hist, krem, sh.scratch + 2 * W);
        __syncthreads();
        prefix = (prefix << width) | sh.scratch[2 * W];
        krem -= (int)sh.scratch[2 * W + 1];
        top = shift;
        if (top > 0 && sh.scratch[2 * W + 2]) {
            const uint32_t edge = lo + (prefix << top);   // lowest key the bin can hold
            if (edge > 0) {
                krem = 0;
                return edge - 1;
            }
        }
    }
    return lo + (prefix << top);
}

// Writes the selected columns of the row, ascending, to stage_col[0, n_out) (and their scores to
// stage_sc when it is given): every column of key > T (all of them when `all`), then per thread in
// column order the ties at T until krem are taken.  Returns n_out (the same in every thread; ends
// with a barrier, so the stage is complete).
template <int NT, int R>
__device__ __forceinline__ int regs_emit(const uint32_t (&key)[R], int c0, int nv, bool all, uint32_t T, int krem,
                                         int k, int32_t* stage_col, float* stage_sc, SelScalars<NT>& sh,
                                         uint32_t* status)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int j = 0; j < R; ++j) {
        if (j >= nv) continue;
        if (all || key[j] > T) gt |= 1u << j;
        else if (key[j] == T) eq |= 1u << j;
    }
    const uint32_t ng = __popc(gt), ne = __popc(eq);
    // exclusive scan of (ng, ne) over the threads, packed in 64 bits
    const uint64_t mine = ((uint64_t)ng << 32) | ne;
    uint64_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    uint64_t* wsum = reinterpret_cast<uint64_t*>(sh.hist);   // NT / 32 <= 32 entries
    __syncthreads();
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    uint64_t before = incl - mine, total = 0;
    for (int w = 0; w < NT / 32; ++w) {
        const uint64_t x = wsum[w];
        if (w < warp) before += x;
        total += x;
    }
    const uint32_t g_before = (uint32_t)(before >> 32), e_before = (uint32_t)before;
    uint32_t out = g_before + min(e_before, (uint32_t)krem);   // ties before this thread are taken first
    int left_e = (int)min(ne, (uint32_t)max(0, krem - (int)e_before));
#pragma unroll
    for (int j = 0; j < R; ++j) {
        bool take = (gt >> j) & 1u;
        if (!take && ((eq >> j) & 1u) && left_e > 0) {
            take = true;
            --left_e;
        }
        if (!take) continue;
        if (DSA_CHECK(out < (uint32_t)k, status, 203)) {   // an output slot of the row
            stage_col[out] = c0 + j;
            if (stage_sc) stage_sc[out] = key_score(key[j]);
        }
        ++out;
    }
    const uint32_t n_gt = (uint32_t)(total >> 32), n_eq = (uint32_t)total;
    __syncthreads();
    return (int)min((uint32_t)k, n_gt + min(n_eq, (uint32_t)krem));
}

// The row's top k as column indices in stage_col[0, n_out), ascending: the load, the radix passes
// (rows of more than k columns) and the emit.
template <int NT, int R>
__device__ __forceinline__ int regs_topk(const float* src, int n, int k, int32_t* stage_col, float* stage_sc,
                                         SelScalars<NT>& sh, uint32_t* status)
{
    uint32_t key[R];
    int c0, nv;
    regs_load<R>(src, n, key, c0, nv);
    const bool all = n <= k;
    int krem = 0;
    uint32_t T = 0;
    if (!all) {
        krem = k;
        T = regs_radix<NT, R>(key, nv, krem, sh);
    }
    return regs_emit<NT, R>(key, c0, nv, all, T, krem, k, stage_col, stage_sc, sh, status);
}

// One CTA per row (rows of at most NT * R columns): the row's top k, ascending, as keys of the
// column map, padded with -1 (and NaN scores) to k.  Dynamic shared memory: k (or 2k with scores)
// 32-bit words.
template <int NT, int R>
__global__ void __launch_bounds__(NT) select_regs_kernel(SelectArgs a)
{
    extern __shared__ __align__(16) int32_t regs_stage[];
    __shared__ SelScalars<NT> sh;
    grid_dep_wait();     // the scores come from the previous kernel
    grid_dep_launch();
    const int r = blockIdx.x;
    if (a.n_rows_dev && r >= *a.n_rows_dev) return;   // uniform exit
    const RowDesc rd = a.rows[r];
    const int k = a.k;
    const float* src = a.S + (int64_t)(a.src_from_list ? rd.list : r) * a.ld_s;
    const int orow = a.out_from_qrow ? rd.qrow : r;
    float* stage_sc = a.out_score ? reinterpret_cast<float*>(regs_stage + k) : nullptr;
    const int n_out = regs_topk<NT, R>(src, rd.ncols, k, regs_stage, stage_sc, sh, a.status);
    int32_t* oidx = a.out_idx + (int64_t)orow * a.ld_idx;
    float* osc = a.out_score ? a.out_score + (int64_t)orow * a.ld_score : nullptr;
    for (int j = threadIdx.x; j < k; j += NT) {
        oidx[j] = j < n_out ? map_col(a.map, rd, regs_stage[j]) : -1;
        if (osc) osc[j] = j < n_out ? stage_sc[j] : __int_as_float(0x7fc00000);
    }
}

// HISA's block stage in one launch per query (block rows: one per query, column c = middle block
// c + 1): the `keep` best middle blocks by register top-k, then the query's kept blocks (block 0,
// those ascending, its own last block; -1 padded to keep + 2), its token row over them and the
// token-scoring work units (`splits` key-tile ranges of the token row).
struct HisaKeptArgs {
    const int32_t* q_pos;
    const int32_t* k_off;
    int32_t B;
    int32_t keep;
    int32_t splits;
    int32_t pad_;
    int32_t* kept;          // [n_q, keep + 2]
    RowDesc* token_rows;    // [n_q]
    TcUnit* units;          // [n_q * splits]
};

template <int NT, int R>
__global__ void __launch_bounds__(NT) hisa_block_select_kernel(SelectArgs a, HisaKeptArgs h)
{
    extern __shared__ __align__(16) int32_t regs_stage[];
    __shared__ SelScalars<NT> sh;
    grid_dep_wait();     // the block scores come from the previous kernel
    grid_dep_launch();
    const int t = blockIdx.x;
    const RowDesc rd = a.rows[t];
    const int n_mid = regs_topk<NT, R>(a.S + (int64_t)t * a.ld_s, rd.ncols, h.keep, regs_stage, nullptr, sh,
                                       a.status);
    const int L = h.k_off[rd.seq + 1] - h.k_off[rd.seq];
    const int n = eligible_count(h.q_pos[t], L);
    const int last = n > 0 ? (n - 1) / h.B : 0;
    const int m = n > 0 ? 1 + n_mid + (last > 0 ? 1 : 0) : 0;   // kept blocks
    int32_t* out = h.kept + (int64_t)t * (h.keep + 2);
    for (int j = threadIdx.x; j < h.keep + 2; j += NT) {
        int32_t v = -1;
        if (j < m) v = j == 0 ? 0 : j <= n_mid ? map_col(a.map, rd, regs_stage[j - 1]) : last;
        out[j] = v;
    }
    const int ncols = m > 0 ? (m - 1) * h.B + (n - last * h.B) : 0;
    if (threadIdx.x == 0) h.token_rows[t] = RowDesc{t, rd.seq, ncols, t};
    const int nkt = (ncols + 127) / 128;
    for (int s = threadIdx.x; s < h.splits; s += NT)
        h.units[(int64_t)t * h.splits + s] =
            TcUnit{t, 1, nkt * s / h.splits, nkt * (s + 1) / h.splits, t, h.k_off[rd.seq], {0, 0}};
}

}  // namespace dsa
