// Exact per-row top-k selection over materialised fp32 score rows.
//
// One CTA ranks one row: a 4-digit (8 bits each) radix select on the
// order-preserving score keys finds the k-th largest key T and how many
// keys equal to T must be taken; an emit pass then writes, in ascending
// column order, every column whose key is above T plus the lowest-indexed
// columns equal to T.  Ties therefore go to the lower key index, which is
// the ranking the indexer pages imply (highest score first) made total.
// Rows up to kSelectSmemKeys columns are staged once in shared memory;
// longer rows are re-read from global memory (L2) on every pass.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kSelectThreads = 512;
constexpr int kSelectWarps = kSelectThreads / 32;
constexpr int kSelectSmemKeys = 40960;   // 160 KB of keys

struct SelectArgs {
    const RowDesc* rows;
    int32_t n_rows;
    int32_t k;
    ColMap map;
    const float* S;          // score row r at S + src_row * ld_s
    int64_t ld_s;
    int32_t src_from_list;   // 1: the score row is rows[r].list instead of r
    int32_t pad_;
    int32_t* out_idx;        // [n_rows, ld_idx]
    int64_t ld_idx;
    float* out_score;        // nullable, [n_rows, ld_score]
    int64_t ld_score;
};

template <bool kSmem>
__global__ void __launch_bounds__(kSelectThreads) select_topk_kernel(SelectArgs a)
{
    extern __shared__ uint32_t skeys[];
    __shared__ uint32_t hist[256];
    __shared__ uint32_t s_bin, s_above;
    __shared__ uint32_t s_gt[kSelectWarps], s_eq[kSelectWarps];

    const int r = blockIdx.x;
    const RowDesc rd = a.rows[r];
    const int n = rd.ncols;
    const int k = a.k;
    const float* src = a.S + (int64_t)(a.src_from_list ? rd.list : r) * a.ld_s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (kSmem) {
        for (int i = tid; i < n; i += kSelectThreads) skeys[i] = score_key(src[i]);
        __syncthreads();
    }
    auto key_at = [&](int i) -> uint32_t { return kSmem ? skeys[i] : score_key(__ldg(src + i)); };

    uint32_t thresh = 0;
    int krem = n;   // n <= k: every column is taken (all keys >= 0)
    if (n > k) {
        uint32_t prefix = 0, mask = 0;
        krem = k;
        const int n_round = (n + 31) & ~31;
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int i = tid; i < 256; i += kSelectThreads) hist[i] = 0;
            __syncthreads();
            for (int i = tid; i < n_round; i += kSelectThreads) {
                const bool valid = i < n;
                const uint32_t u = valid ? key_at(i) : 0u;
                const bool in = valid && ((u & mask) == prefix);
                const uint32_t bin = (u >> shift) & 255u;
                const uint32_t active = __ballot_sync(0xffffffffu, in);
                if (in) {
                    const uint32_t peers = __match_any_sync(active, bin);
                    if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
                }
            }
            __syncthreads();
            if (warp == 0) {
                // lane l owns bins 8l .. 8l+7; counts from the top decide the bin holding rank krem
                uint32_t c[8], tot = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) { c[j] = hist[8 * lane + j]; tot += c[j]; }
                uint32_t incl = tot;   // sum over lanes >= lane
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const uint32_t v = __shfl_down_sync(0xffffffffu, incl, off);
                    if (lane + off < 32) incl += v;
                }
                const uint32_t above = incl - tot;
                if (above < (uint32_t)krem && (uint32_t)krem <= incl) {
                    uint32_t acc = above;
                    int b = 0;
#pragma unroll
                    for (int j = 7; j >= 0; --j) {
                        if (acc + c[j] >= (uint32_t)krem) { b = j; break; }
                        acc += c[j];
                    }
                    s_bin = 8 * lane + b;
                    s_above = acc;
                }
            }
            __syncthreads();
            prefix |= s_bin << shift;
            mask |= 255u << shift;
            krem -= (int)s_above;
            __syncthreads();
        }
        thresh = prefix;
    }

    // Emit: warp w owns the contiguous columns [w*seg, (w+1)*seg).
    const int seg = ((n + kSelectWarps - 1) / kSelectWarps + 31) & ~31;
    const int beg = warp * seg;
    const int end = min(beg + seg, n);
    uint32_t gt = 0, eq = 0;
    for (int base = beg; base < end; base += 32) {
        const int i = base + lane;
        const bool v = i < end;
        const uint32_t u = v ? key_at(i) : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, v && u > thresh));
        eq += __popc(__ballot_sync(0xffffffffu, v && u == thresh));
    }
    if (lane == 0) { s_gt[warp] = gt; s_eq[warp] = eq; }
    __syncthreads();
    uint32_t gt_before = 0, eq_before = 0;
    for (int w = 0; w < warp; ++w) { gt_before += s_gt[w]; eq_before += s_eq[w]; }
    uint32_t out = gt_before + min(eq_before, (uint32_t)krem);
    uint32_t eq_rank = eq_before;
    int32_t* oidx = a.out_idx + (int64_t)r * a.ld_idx;
    float* osc = a.out_score ? a.out_score + (int64_t)r * a.ld_score : nullptr;
    for (int base = beg; base < end; base += 32) {
        const int i = base + lane;
        const bool v = i < end;
        const uint32_t u = v ? key_at(i) : 0u;
        const bool is_gt = v && u > thresh;
        const bool is_eq = v && u == thresh;
        const uint32_t eqb = __ballot_sync(0xffffffffu, is_eq);
        const uint32_t my_rank = eq_rank + __popc(eqb & lanemask_lt());
        const bool emit = is_gt || (is_eq && my_rank < (uint32_t)krem);
        const uint32_t eb = __ballot_sync(0xffffffffu, emit);
        if (emit) {
            const uint32_t o = out + __popc(eb & lanemask_lt());
            oidx[o] = map_col(a.map, rd, i);
            if (osc) osc[o] = key_score(u);
        }
        out += __popc(eb);
        eq_rank += __popc(eqb);
    }
    const int n_out = min(n, k);
    for (int j = n_out + tid; j < k; j += kSelectThreads) {
        oidx[j] = -1;
        if (osc) osc[j] = __int_as_float(0x7fc00000);
    }
}

}  // namespace dsa
