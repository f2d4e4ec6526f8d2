// Exact per-row top-k selection over fp32 score rows in global memory.
//
// The result of a row is every column whose score key is above T (the k-th
// largest key of the row) plus the lowest columns whose key equals T: ties
// go to the lower key index.  Columns are written in ascending order.
//
// One CTA of 256 threads ranks one row, keeping little state so several rows
// are in flight per SM:
//   1. threshold: the keys of 2048 evenly spaced columns are ranked and the
//      one at rank k*m/n plus a 4-sigma margin becomes tau (rows with at most
//      select_buf_cap(k) columns skip this and keep every column);
//   2. one streaming pass appends every column with key >= tau to a
//      shared-memory buffer (select_buf_cap(k) entries);
//   3. if at least k columns passed and none was dropped, the top k of the
//      row are exactly the top k of the buffer: an 8-bit radix select over
//      the buffer finds T and the number of T-ties to take.  Otherwise
//      (a misleading sample) T is found by radix passes over the whole row;
//   4. the selected columns are marked in two bitmaps (> T, == T) and emitted
//      in column order, taking the first ties.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSampleMax = 2048;

// Candidate buffer entries for top-k: at least 4096 and 1.75 k.
__host__ __device__ inline int select_buf_cap(int k)
{
    const int c = (7 * k / 4 + 255) & ~255;
    return c < 4096 ? 4096 : c;
}

struct SelectArgs {
    const RowDesc* rows;
    int32_t n_rows;
    int32_t k;
    ColMap map;
    const float* S;          // score row r at S + src_row * ld_s
    int64_t ld_s;
    int32_t src_from_list;   // 1: the score row is rows[r].list instead of r
    int32_t buf_cap;         // candidate buffer entries (select_stream_kernel)
    int32_t* out_idx;        // [n_rows, ld_idx]
    int64_t ld_idx;
    float* out_score;        // nullable, [n_rows, ld_score]
    int64_t ld_score;
};


// Dynamic shared memory of select_stream_kernel for rows of up to max_cols columns.
__host__ __device__ inline size_t select_smem_bytes(int max_cols, int buf_cap)
{
    const size_t words = (size_t)(max_cols + 31) / 32;
    return kSampleMax * 4 + (size_t)buf_cap * 8 + 2 * words * 4;
}

// Exact rank selection among `count` keys given by get(i): returns the key T
// holding rank `krem` (1 = largest) and, in krem, how many keys equal to T
// that rank reaches.  Digits are taken from (key - min), starting at the
// highest bit where min and max differ, 8 bits at a time, so even the first
// pass spreads the keys over many bins.  All threads call it.
template <int NT, typename Get>
__device__ __forceinline__ uint32_t radix_select(Get get, int count, int& krem, uint32_t* hist, uint32_t* scratch)
{
    constexpr int kSelThreads = NT;
    constexpr int kSelWarps = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int i = tid; i < count; i += kSelThreads) {
        const uint32_t u = get(i);
        lo = min(lo, u);
        hi = max(hi, u);
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    __syncthreads();
    if (lane == 0) { scratch[warp] = lo; scratch[kSelWarps + warp] = hi; }
    __syncthreads();
    lo = scratch[0];
    hi = scratch[kSelWarps];
#pragma unroll
    for (int w = 1; w < kSelWarps; ++w) { lo = min(lo, scratch[w]); hi = max(hi, scratch[kSelWarps + w]); }
    int top = 32 - __clz(hi - lo);   // bits of (key - lo) still undecided
    uint32_t prefix = 0;             // decided high bits of (T - lo)
    while (top > 0) {
        const int shift = max(top - 8, 0), width = top - shift;
        __syncthreads();
        for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < count; i += kSelThreads) {
            const uint32_t rel = get(i) - lo;
            if ((uint32_t)((uint64_t)rel >> top) == prefix) atomicAdd(&hist[(rel >> shift) & ((1u << width) - 1u)], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t c[8], tot = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) { c[b] = hist[8 * lane + b]; tot += c[b]; }
            uint32_t incl = tot;   // keys in the digits of lanes >= this lane
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t x = __shfl_down_sync(0xffffffffu, incl, o);
                if (lane + o < 32) incl += x;
            }
            const uint32_t above = incl - tot;
            if (above < (uint32_t)krem && (uint32_t)krem <= incl) {
                uint32_t acc = above;
                int b = 7;
                for (; b > 0; --b) {
                    if (acc + c[b] >= (uint32_t)krem) break;
                    acc += c[b];
                }
                scratch[2 * kSelWarps] = 8 * lane + b;
                scratch[2 * kSelWarps + 1] = acc;
            }
        }
        __syncthreads();
        prefix = (prefix << width) | scratch[2 * kSelWarps];
        krem -= (int)scratch[2 * kSelWarps + 1];
        top = shift;
    }
    return lo + prefix;
}

template <int NT>
__global__ void __launch_bounds__(NT) select_stream_kernel(SelectArgs a)
{
    constexpr int kSelThreads = NT;
    constexpr int kSelWarps = NT / 32;
    extern __shared__ __align__(16) uint8_t sel_smem[];
    uint32_t* sample = reinterpret_cast<uint32_t*>(sel_smem);
    const int kBufCap = a.buf_cap;
    uint64_t* buf = reinterpret_cast<uint64_t*>(sel_smem + kSampleMax * 4);
    uint32_t* gtmap = reinterpret_cast<uint32_t*>(sel_smem + kSampleMax * 4 + (size_t)kBufCap * 8);
    __shared__ uint32_t hist[256];
    __shared__ uint32_t scratch[2 * kSelWarps + 2];
    __shared__ uint32_t s_count;
    __shared__ uint32_t s_wgt[kSelWarps], s_weq[kSelWarps];

    const int r = blockIdx.x;
    const RowDesc rd = a.rows[r];
    const int n = rd.ncols;
    const int k = a.k;
    const float* src = a.S + (int64_t)(a.src_from_list ? rd.list : r) * a.ld_s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwords = (n + 31) >> 5;
    uint32_t* eqmap = gtmap + nwords;
    int32_t* oidx = a.out_idx + (int64_t)r * a.ld_idx;
    float* osc = a.out_score ? a.out_score + (int64_t)r * a.ld_score : nullptr;

    for (int w = tid; w < 2 * nwords; w += kSelThreads) gtmap[w] = 0;
    uint32_t thresh = 0;   // T: the k-th largest key (0 when every column is taken)
    int krem = n;          // ties at T still to take
    if (n > k) {
        // ---- 1. threshold from a sample (or every column for short rows)
        uint32_t tau = 0;
        if (n > kBufCap) {
            const int m = kSampleMax;
            float x[kSampleMax / kSelThreads];   // all sample loads in flight at once
#pragma unroll
            for (int j = 0; j < kSampleMax / kSelThreads; ++j)
                x[j] = __ldg(src + (int)(((int64_t)(tid + j * kSelThreads) * n) / m));
#pragma unroll
            for (int j = 0; j < kSampleMax / kSelThreads; ++j) sample[tid + j * kSelThreads] = score_key(x[j]);
            const float expect = (float)k * m / n;
            int rank = (int)ceilf(expect + 4.f * sqrtf(expect) + 4.f);
            rank = min(rank, m);
            __syncthreads();
            tau = radix_select<NT>([&](int i) { return sample[i]; }, m, rank, hist, scratch);
        }
        // ---- 2. one pass: every column with key >= tau into the buffer
        if (tid == 0) s_count = 0;
        __syncthreads();
        // Appends the columns of this lane that pass, one shared atomic per warp.
        // nv: how many of x's four columns (c .. c+3) exist.
        auto keep4 = [&](float4 x, int c, int nv) {
            const uint32_t u0 = score_key(x.x), u1 = score_key(x.y), u2 = score_key(x.z), u3 = score_key(x.w);
            const bool p0 = nv > 0 && u0 >= tau, p1 = nv > 1 && u1 >= tau, p2 = nv > 2 && u2 >= tau,
                       p3 = nv > 3 && u3 >= tau;
            const uint32_t b0 = __ballot_sync(0xffffffffu, p0), b1 = __ballot_sync(0xffffffffu, p1);
            const uint32_t b2 = __ballot_sync(0xffffffffu, p2), b3 = __ballot_sync(0xffffffffu, p3);
            const uint32_t total = __popc(b0) + __popc(b1) + __popc(b2) + __popc(b3);
            if (total == 0) return;
            uint32_t slot = 0;
            if (lane == 0) slot = atomicAdd(&s_count, total);
            slot = __shfl_sync(0xffffffffu, slot, 0);
            const uint32_t lt = lanemask_lt();
            uint32_t o = slot + __popc(b0 & lt);
            if (p0 && o < (uint32_t)kBufCap) buf[o] = ((uint64_t)u0 << 32) | (uint32_t)c;
            o = slot + __popc(b0) + __popc(b1 & lt);
            if (p1 && o < (uint32_t)kBufCap) buf[o] = ((uint64_t)u1 << 32) | (uint32_t)(c + 1);
            o = slot + __popc(b0) + __popc(b1) + __popc(b2 & lt);
            if (p2 && o < (uint32_t)kBufCap) buf[o] = ((uint64_t)u2 << 32) | (uint32_t)(c + 2);
            o = slot + __popc(b0) + __popc(b1) + __popc(b2) + __popc(b3 & lt);
            if (p3 && o < (uint32_t)kBufCap) buf[o] = ((uint64_t)u3 << 32) | (uint32_t)(c + 3);
        };
        const bool vec = (reinterpret_cast<uintptr_t>(src) & 15) == 0;
        const int n4 = vec ? (n >> 2) : 0;
        const float4* s4 = reinterpret_cast<const float4*>(src);
        constexpr int U = 8;   // 16-byte loads in flight per thread
        for (int c4 = warp * 32; c4 < n4; c4 += U * kSelThreads) {   // warp-uniform trip count
            float4 x[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = c4 + u * kSelThreads + lane;
                x[u] = i < n4 ? __ldg(s4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = c4 + u * kSelThreads + lane;
                keep4(x[u], 4 * i, i < n4 ? 4 : 0);
            }
        }
        for (int c0 = 4 * n4 + warp * 32; c0 < n; c0 += kSelThreads) {   // tail (or the whole row if unaligned)
            const int c = c0 + lane;
            const float v0 = c < n ? __ldg(src + c) : 0.f;
            keep4(make_float4(v0, 0.f, 0.f, 0.f), c, c < n ? 1 : 0);
        }
        __syncthreads();
        const int count = (int)s_count;
        krem = k;
        if (count >= k && count <= kBufCap) {
            // ---- 3. exact top-k of the buffer
            thresh = radix_select<NT>([&](int i) { return (uint32_t)(buf[i] >> 32); }, count, krem, hist, scratch);
            for (int i = tid; i < count; i += kSelThreads) {
                const uint32_t u = (uint32_t)(buf[i] >> 32), c = (uint32_t)buf[i];
                if (u > thresh) atomicOr(&gtmap[c >> 5], 1u << (c & 31));
                else if (u == thresh) atomicOr(&eqmap[c >> 5], 1u << (c & 31));
            }
        } else {
            // ---- 3'. the sample misled: exact selection over the whole row
            thresh = radix_select<NT>([&](int i) { return score_key(__ldg(src + i)); }, n, krem, hist, scratch);
            for (int c = tid; c < n; c += kSelThreads) {
                const uint32_t u = score_key(__ldg(src + c));
                if (u > thresh) atomicOr(&gtmap[c >> 5], 1u << (c & 31));
                else if (u == thresh) atomicOr(&eqmap[c >> 5], 1u << (c & 31));
            }
        }
    } else {
        __syncthreads();
        for (int w = tid; w < nwords; w += kSelThreads)
            gtmap[w] = (w + 1) * 32 <= n ? 0xffffffffu : ((1u << (n & 31)) - 1u);
    }
    __syncthreads();

    // ---- 4. emit in column order: warp w owns words [w*wpw, (w+1)*wpw)
    const int wpw = (nwords + kSelWarps - 1) / kSelWarps;
    const int w0 = warp * wpw, w1 = min(w0 + wpw, nwords);
    uint32_t gt = 0, eq = 0;
    for (int w = w0 + lane; w < w1; w += 32) { gt += __popc(gtmap[w]); eq += __popc(eqmap[w]); }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        gt += __shfl_xor_sync(0xffffffffu, gt, o);
        eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (lane == 0) { s_wgt[warp] = gt; s_weq[warp] = eq; }
    __syncthreads();
    uint32_t eq_rank = 0, out = 0;
    for (int w = 0; w < warp; ++w) { out += s_wgt[w]; eq_rank += s_weq[w]; }
    out += min(eq_rank, (uint32_t)krem);
    for (int wb = w0; wb < w1; wb += 32) {
        const int w = wb + lane;
        const uint32_t g = w < w1 ? gtmap[w] : 0u, e = w < w1 ? eqmap[w] : 0u;
        const uint32_t ce = __popc(e);
        uint32_t pre_e = ce;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, pre_e, o);
            if (lane >= o) pre_e += x;
        }
        const uint32_t rank0 = eq_rank + pre_e - ce;   // ties before this word
        const int n_take_e = (int)min(ce, (uint32_t)max(0, krem - (int)rank0));
        uint32_t take_e = e;
        for (int drop = (int)ce - n_take_e; drop > 0; --drop) take_e &= ~(1u << (31 - __clz(take_e)));   // keep lowest
        const uint32_t take = g | take_e;
        const uint32_t ct = __popc(take);
        uint32_t pre_t = ct;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, pre_t, o);
            if (lane >= o) pre_t += x;
        }
        uint32_t o = out + pre_t - ct;
        for (uint32_t bits = take; bits; bits &= bits - 1) {
            const int col = w * 32 + __ffs(bits) - 1;
            oidx[o] = map_col(a.map, rd, col);
            if (osc) osc[o] = key_score(score_key(__ldg(src + col)));
            ++o;
        }
        out += __shfl_sync(0xffffffffu, pre_t, 31);
        eq_rank += __shfl_sync(0xffffffffu, pre_e, 31);
    }
    const int n_out = min(n, k);
    for (int j = n_out + tid; j < k; j += kSelThreads) {
        oidx[j] = -1;
        if (osc) osc[j] = __int_as_float(0x7fc00000);
    }
}

}  // namespace dsa
