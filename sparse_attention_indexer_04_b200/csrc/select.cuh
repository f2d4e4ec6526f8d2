// Exact per-row top-k selection over fp32 score rows in global memory.
//
// The result of a row is every column whose score key is above T (the k-th
// largest key of the row) plus the lowest columns whose key equals T: ties
// go to the lower key index.  Columns are written in ascending order.
//
// A row is ranked in four steps (the CTA first starts a bulk L2 prefetch of
// its row, so that step 2 reads L2):
//   1. threshold: the keys of m columns (m >= 128 n / k, 2048 to 8192), in
//      m/32 evenly spaced runs of 32, are ranked and the one at rank k*m/n
//      plus a 4-sigma margin becomes tau (rows that fit the candidate buffer
//      skip this and keep every column);
//   2. one streaming pass appends every column with key >= tau (tested on
//      the float itself) to a candidate buffer of about 1.75 k entries, as
//      (score bits, column);
//   3. if at least k columns passed and none was dropped, the top k of the
//      row are exactly the top k of the buffer: its scores become keys and
//      an 8-bit radix select over it finds T and the number of T-ties to
//      take.  Otherwise (a misleading sample) T is found by radix passes
//      over the whole row;
//   4. the selected columns are marked in two bitmaps (> T, == T) and emitted
//      in column order, taking the first ties; the output row is assembled in
//      shared memory and written with 16-byte stores.
// select_stream_kernel gives each row one CTA (many rows: prefill).
// select_split_kernel gives each row several CTAs that share step 2 through
// a global buffer, the last of them finishing the row (few long rows: decode).
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace dsa {

constexpr int kSampleMin = 2048;
constexpr int kSampleMax = 8192;

// Sample size for a row of n columns and rank k: enough that the expected rank of the k-th
// largest key in the sample, k * m / n, is 128 or more (the candidate count then stays within
// the 1.75 k buffer by several standard deviations), in multiples of 2048, 2048 to 8192.
__host__ __device__ inline int select_sample_size(int n, int k)
{
    const int64_t need = (128 * (int64_t)n + k - 1) / (k > 0 ? k : 1);
    const int64_t m = (need + kSampleMin - 1) / kSampleMin * kSampleMin;
    return m < kSampleMin ? kSampleMin : (m > kSampleMax ? kSampleMax : (int)m);
}

// A smaller sample for rows of up to 256K columns: at most 4096, the candidate buffer sized for the
// wider threshold.  Every CTA of the cluster select ranks the whole sample; the one-CTA select takes
// it for long rows (PIVOT's group lists over 128K proxy rows).
__host__ __device__ inline int capped_sample_size(int n, int k)
{
    const int m = select_sample_size(n, k);
    return n <= 262144 && m > 4096 ? 4096 : m;
}

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
    int32_t buf_cap;         // candidate buffer entries
    int32_t sample_bytes;    // shared memory of the sample: select_sample_bytes(max_cols, k)
    int32_t* out_idx;        // [n_rows, ld_idx]
    int64_t ld_idx;
    float* out_score;        // nullable, [n_rows, ld_score]
    int64_t ld_score;
    const int32_t* n_rows_dev;   // nullable: rows [*n_rows_dev, n_rows) are skipped (a count a kernel wrote)
    int32_t out_from_qrow;       // 1: row r writes output row rows[r].qrow instead of r
    int32_t capped_sample;       // 1: the one-CTA select samples capped_sample_size columns (long rows)
    uint32_t* status;            // the workspace status word (checked builds record index errors there)
};


// Dynamic shared memory of the select kernels for rows of up to max_cols columns: the sample, the
// candidate buffer and two bitmaps of the row's columns.
__host__ __device__ inline size_t select_sample_bytes(int max_cols, int k)
{
    return (size_t)select_sample_size(max_cols, k) * 4;
}

__host__ __device__ inline size_t select_smem_bytes(int max_cols, int buf_cap, int k)
{
    const size_t words = (size_t)(max_cols + 31) / 32;
    return select_sample_bytes(max_cols, k) + (size_t)buf_cap * 8 + 2 * words * 4;
}

// Block-wide min and max of the keys each thread passes in (lo, hi): every thread gets the result.
// Ends with a barrier, so shared-memory writes made before the call are visible after it.
template <int NT>
__device__ __forceinline__ void block_key_range(uint32_t& lo, uint32_t& hi, uint32_t* scratch)
{
    constexpr int kSelWarps = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    __syncthreads();
    if (lane == 0) { scratch[warp] = lo; scratch[kSelWarps + warp] = hi; }
    __syncthreads();
    lo = scratch[0];
    hi = scratch[kSelWarps];
#pragma unroll
    for (int w = 1; w < kSelWarps; ++w) { lo = min(lo, scratch[w]); hi = max(hi, scratch[kSelWarps + w]); }
}

// Run by one warp after a radix pass: finds the bin of the 256-bin histogram that holds rank krem
// (1 = largest) and writes out[0] = the bin, out[1] = the keys in the bins above it, out[2] = 1 when
// the bin's keys are all taken (rank krem is its lowest key).
__device__ __forceinline__ void radix_pick(const uint32_t* hist, int krem, uint32_t* out)
{
    const int lane = threadIdx.x & 31;
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
        out[0] = 8 * lane + b;
        out[1] = acc;
        out[2] = acc + c[b] == (uint32_t)krem;   // the whole bin is taken
    }
}

// Exact rank selection among `count` keys given by get(i): returns the key T
// holding rank `krem` (1 = largest) and, in krem, how many keys equal to T
// that rank reaches.  Digits are taken from (key - min), starting at the
// highest bit where min and max differ, 8 bits at a time, so even the first
// pass spreads the keys over many bins.  When the rank falls in a bin whose
// keys are all taken, the passes stop there and the result says "every key
// >= the bin's lower edge": T = that edge - 1 and krem = 0 (no tie at T is
// taken).  With stop_bits > 0 only the top stop_bits bits of (key - min) are
// resolved and the lower edge of that bin is returned: a key <= T (krem is
// then meaningless).  All threads call it.
//
// radix_select with the keys' block-wide range [lo, hi] already known (all threads pass the same).
template <int NT, typename Get>
__device__ __forceinline__ uint32_t radix_select_in(Get get, int count, int& krem, uint32_t lo, uint32_t hi,
                                                    uint32_t* hist, uint32_t* scratch, int stop_bits = 0)
{
    constexpr int kSelThreads = NT;
    constexpr int kSelWarps = NT / 32;
    const int tid = threadIdx.x, warp = tid >> 5;
    int top = 32 - __clz(hi - lo);   // bits of (key - lo) still undecided
    const int stop = stop_bits > 0 ? max(top - stop_bits, 0) : 0;
    uint32_t prefix = 0;             // decided high bits of (T - lo)
    while (top > stop) {
        const int shift = max(top - 8, 0), width = top - shift;
        __syncthreads();
        for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < count; i += kSelThreads) {
            const uint32_t rel = get(i) - lo;
            if (((rel >> 1) >> (top - 1)) == prefix) atomicAdd(&hist[(rel >> shift) & ((1u << width) - 1u)], 1u);
        }
        __syncthreads();
        if (warp == 0) radix_pick(hist, krem, scratch + 2 * kSelWarps);
        __syncthreads();
        prefix = (prefix << width) | scratch[2 * kSelWarps];
        krem -= (int)scratch[2 * kSelWarps + 1];
        top = shift;
        if (stop_bits == 0 && top > 0 && scratch[2 * kSelWarps + 2]) {
            const uint32_t edge = lo + (prefix << top);   // lowest key the bin can hold
            if (edge > 0) {
                krem = 0;
                return edge - 1;
            }
        }
    }
    return lo + (prefix << top);
}

template <int NT, typename Get>
__device__ __forceinline__ uint32_t radix_select(Get get, int count, int& krem, uint32_t* hist, uint32_t* scratch,
                                                 int stop_bits = 0)
{
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int i = threadIdx.x; i < count; i += NT) {
        const uint32_t u = get(i);
        lo = min(lo, u);
        hi = max(hi, u);
    }
    block_key_range<NT>(lo, hi, scratch);
    return radix_select_in<NT>(get, count, krem, lo, hi, hist, scratch, stop_bits);
}

// Starts bringing the scores [p, p + count) into L2 while the row's first steps run (the candidate
// scan then reads L2 instead of waiting on DRAM): 64 KB pieces, one per thread of the first few.
// Skipped for rows not 16-byte aligned; the last partial 16 bytes are left out.
__device__ __forceinline__ void prefetch_row_l2(const float* p, int64_t count)
{
    if ((reinterpret_cast<uintptr_t>(p) & 15) != 0) return;
    const int64_t bytes = (count * 4) & ~15ll;
    constexpr int64_t kPiece = 65536;
    const int64_t off = (int64_t)threadIdx.x * kPiece;
    if (off < bytes) prefetch_l2_bulk(reinterpret_cast<const char*>(p) + off, (uint32_t)min(kPiece, bytes - off));
}

// Shared scalars of one selection CTA.
template <int NT>
struct alignas(16) SelScalars {
    uint32_t hist[256];   // radix histogram; the emit step reuses it for per-warp 64-bit sums
    uint32_t scratch[2 * (NT / 32) + 4];
    uint32_t count;   // candidates seen by the append pass
    uint32_t base;    // split rows: this CTA's first slot in the row's global buffer
    uint32_t last;    // split rows: this CTA finishes the row
};

// 1. tau for a row of n > k columns: 0 (every column is a candidate) when n <= buf_cap, else
// the key at rank expect + 4 sqrt(expect) + 4 among m = select_sample_size(n, k) sampled
// columns, expect = k * m / n (the expected rank of the k-th largest key in the sample, plus a
// margin).
template <int NT>
__device__ __forceinline__ uint32_t sel_threshold(const float* src, int n, int k, int buf_cap, uint32_t* sample,
                                                  SelScalars<NT>& sh, int m_given = 0)
{
    if (n <= buf_cap) return 0u;
    static_assert(NT >= 256 && kSampleMax / NT <= 32, "one run start per lane");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m = m_given > 0 ? m_given : select_sample_size(n, k);   // a multiple of 2048
    // m / 32 evenly spaced runs of 32 consecutive columns (a warp reads one run: one or two cache
    // lines instead of 32 scattered sectors); run r starts at floor(r n / R) rounded down to 32.
    // Sample entry e belongs to run e / 32, so a warp's i-th run is warp + i NT / 32; lane i
    // computes that run's start once (r n < 2^31: 32-bit arithmetic) and the loads fetch it by shuffle.
    const uint32_t R = (uint32_t)(m / 32);
    const uint32_t my_run = (uint32_t)(warp + lane * (NT / 32));
    const int my_start = my_run < R ? (int)(((my_run * (uint32_t)n) / R) & ~31u) : 0;
    constexpr int J = kSampleMin / NT;     // sample loads in flight per thread
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int j0 = 0; j0 < m; j0 += kSampleMin) {
        float x[J];
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int col = __shfl_sync(0xffffffffu, my_start, j0 / NT + j) + lane;
            x[j] = __ldg(src + min(col, n - 1));   // runs narrower than 32 columns (n < 32 R) stop at the row's end
        }
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const uint32_t u = score_key(x[j]);
            sample[j0 + tid + j * NT] = u;
            lo = min(lo, u);
            hi = max(hi, u);
        }
    }
    const float expect = (float)k * m / n;
    int rank = (int)ceilf(expect + 4.f * sqrtf(expect) + 4.f);
    rank = min(rank, m);
    block_key_range<NT>(lo, hi, sh.scratch);   // its barriers also publish the sample
    // 16 bits of the sample's key range are enough: the bin's lower edge only lowers tau a little
    return radix_select_in<NT>([&](int i) { return sample[i]; }, m, rank, lo, hi, sh.hist, sh.scratch, 16);
}

// 2. Appends (score bits << 32 | column) of every column c in [c0, c1) whose key is >= max(tau, 1)
// to buf; sh.count (zero on entry) counts them all, entries past cap are dropped.  (Key 0 is a
// NaN with every bit set; leaving it out keeps the buffer exact: with k entries or more, the
// k-th largest is >= 1.)  The test is made on the float itself against the float whose key is
// max(tau, 1) (-inf when that key is at or below -inf's): for every non-NaN score the two agree,
// -0 and +0 included.  sel_buf_keys turns the stored scores into keys.  c0 is a multiple of 4.
// Each thread loads 16 columns per round; a warp finds its threads' output offsets by one prefix
// count over the threads' pass counts (five ballots on the count's bits), takes one shared
// atomic, and each thread writes its passing columns at consecutive slots.
template <int NT>
__device__ __forceinline__ void sel_append(const float* src, int c0, int c1, uint32_t tau, uint64_t* buf, int cap,
                                           SelScalars<NT>& sh)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t t1 = max(tau, 1u);
    const float tf = t1 <= 0x007fffffu ? -INFINITY : key_score(t1);   // 0x007fffff: the key of -inf
    const uint32_t lt = lanemask_lt();
    // A warp's slots for `cnt` entries of this lane (cnt < 32), in lane order; returns the first.
    auto warp_slots = [&](uint32_t cnt, uint32_t& total) {
        uint32_t excl = 0;
        total = 0;
#pragma unroll
        for (int b = 0; b < 5; ++b) {
            const uint32_t bb = __ballot_sync(0xffffffffu, (cnt >> b) & 1u);
            excl += __popc(bb & lt) << b;
            total += __popc(bb) << b;
        }
        uint32_t slot = 0;
        if (total != 0) {
            if (lane == 0) slot = atomicAdd(&sh.count, total);
            slot = __shfl_sync(0xffffffffu, slot, 0);
        }
        return slot + excl;
    };
    const float* s = src + c0;
    const int len = c1 - c0;
    const bool vec = (reinterpret_cast<uintptr_t>(s) & 15) == 0;
    const int n4 = vec ? (len >> 2) : 0;
    const float4* s4 = reinterpret_cast<const float4*>(s);
    constexpr int U = 4;   // 16-byte loads in flight per thread
    for (int i4 = warp * 32; i4 < n4; i4 += U * NT) {   // warp-uniform trip count
        float4 x[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i4 + u * NT + lane;
            x[u] = i < n4 ? __ldg(s4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float v[U][4];
        uint32_t cnt = 0;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const bool ok = i4 + u * NT + lane < n4;
            v[u][0] = x[u].x; v[u][1] = x[u].y; v[u][2] = x[u].z; v[u][3] = x[u].w;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (!ok) v[u][e] = __int_as_float(0x7fffffff);   // NaN: never passes
                cnt += v[u][e] >= tf;
            }
        }
        uint32_t total;
        uint32_t o = warp_slots(cnt, total);
        if (total == 0) continue;
        const uint32_t col0 = (uint32_t)(c0 + 4 * (i4 + lane));
        if (o + cnt <= (uint32_t)cap) {
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const bool pass = v[u][e] >= tf;
                    if (pass) buf[o] = ((uint64_t)__float_as_uint(v[u][e]) << 32) | (col0 + 4 * u * NT + e);
                    o += pass;
                }
        } else {
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const bool pass = v[u][e] >= tf;
                    if (pass && o < (uint32_t)cap)
                        buf[o] = ((uint64_t)__float_as_uint(v[u][e]) << 32) | (col0 + 4 * u * NT + e);
                    o += pass;
                }
        }
    }
    for (int j0 = 4 * n4 + warp * 32; j0 < len; j0 += NT) {   // tail (or the whole range if unaligned)
        const int j = j0 + lane;
        const float v0 = j < len ? __ldg(s + j) : __int_as_float(0x7fffffff);
        const bool pass = v0 >= tf;
        uint32_t total;
        const uint32_t o = warp_slots(pass ? 1u : 0u, total);
        if (pass && o < (uint32_t)cap) buf[o] = ((uint64_t)__float_as_uint(v0) << 32) | (uint32_t)(c0 + j);
    }
}

// Turns the buffer's first count entries from (score bits, column) into (key, column) and returns
// the keys' block-wide range (every thread; ends with a barrier).
template <int NT>
__device__ __forceinline__ void sel_buf_keys(uint64_t* buf, int count, uint32_t& lo, uint32_t& hi,
                                             SelScalars<NT>& sh)
{
    lo = 0xffffffffu;
    hi = 0u;
    for (int i = threadIdx.x; i < count; i += NT) {
        const uint64_t e = buf[i];
        const uint32_t u = score_key(__uint_as_float((uint32_t)(e >> 32)));
        buf[i] = ((uint64_t)u << 32) | (uint32_t)e;
        lo = min(lo, u);
        hi = max(hi, u);
    }
    block_key_range<NT>(lo, hi, sh.scratch);
}

// 3. Marks the row's top k in the bitmaps (> T in gtmap, == T in eqmap, both zeroed) and returns
// in krem how many ties at T to take.  From the candidate buffer (score bits, turned into keys
// here) when it holds every column with key >= tau (k <= count <= cap), else (a misleading
// sample) by radix passes over the whole row.
template <int NT>
__device__ __forceinline__ void sel_mark(const float* src, int n, int k, uint64_t* buf, int count, int cap,
                                         int& krem, uint32_t* gtmap, uint32_t* eqmap, SelScalars<NT>& sh,
                                         uint32_t* status = nullptr)
{
    const int tid = threadIdx.x;
    krem = k;
    if (count >= k && count <= cap) {
        uint32_t lo, hi;
        sel_buf_keys<NT>(buf, count, lo, hi, sh);
        const uint32_t thresh = radix_select_in<NT>([&](int i) { return (uint32_t)(buf[i] >> 32); }, count, krem,
                                                    lo, hi, sh.hist, sh.scratch);
        for (int i = tid; i < count; i += NT) {
            const uint32_t u = (uint32_t)(buf[i] >> 32), c = (uint32_t)buf[i];
            if (!DSA_CHECK(c < (uint32_t)n, status, 201)) continue;   // a candidate column of the row
            if (u > thresh) atomicOr(&gtmap[c >> 5], 1u << (c & 31));
            else if (u == thresh) atomicOr(&eqmap[c >> 5], 1u << (c & 31));
        }
    } else {
        const uint32_t thresh =
            radix_select<NT>([&](int i) { return score_key(__ldg(src + i)); }, n, krem, sh.hist, sh.scratch);
        for (int c = tid; c < n; c += NT) {
            const uint32_t u = score_key(__ldg(src + c));
            if (u > thresh) atomicOr(&gtmap[c >> 5], 1u << (c & 31));
            else if (u == thresh) atomicOr(&eqmap[c >> 5], 1u << (c & 31));
        }
    }
}

// Rows of at most k columns: every column is taken.
template <int NT>
__device__ __forceinline__ void sel_mark_all(int n, uint32_t* gtmap)
{
    const int nwords = (n + 31) >> 5;
    for (int w = threadIdx.x; w < nwords; w += NT)
        gtmap[w] = (w + 1) * 32 <= n ? 0xffffffffu : ((1u << (n & 31)) - 1u);
}

// 4. Emits the marked columns in column order (all of gtmap, the first krem of eqmap), then pads
// the row to k with -1 (and NaN scores).  Thread t owns a contiguous run of bitmap words; one
// block-wide scan of its (> T, == T) counts gives both its output offset and its tie rank.  When
// the row fits in stage (16-byte aligned, stage_words words: k, or 2k with scores, whose columns are
// staged and read back all at once) it is assembled
// there and written with coalesced 16-byte stores, else written directly.
template <int NT>
__device__ __forceinline__ void sel_emit(const SelectArgs& a, const RowDesc& rd, int r, const float* src, int n,
                                         int krem, const uint32_t* gtmap, const uint32_t* eqmap, int32_t* stage,
                                         int stage_words, SelScalars<NT>& sh)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = a.k;
    const int nwords = (n + 31) >> 5;
    int32_t* oidx = a.out_idx + (int64_t)r * a.ld_idx;
    float* osc = a.out_score ? a.out_score + (int64_t)r * a.ld_score : nullptr;
    const bool staged = (osc ? 2 * k : k) <= stage_words;
    const int wpt = (nwords + NT - 1) / NT;
    const int w0 = min(nwords, tid * wpt), w1 = min(nwords, w0 + wpt);
    uint32_t ng = 0, ne = 0;
    for (int w = w0; w < w1; ++w) { ng += __popc(gtmap[w]); ne += __popc(eqmap[w]); }
    // exclusive scan of (ng, ne) over the threads, packed in 64 bits (each sum < 2^32)
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
    uint64_t before = incl - mine;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    const uint32_t g_before = (uint32_t)(before >> 32), e_before = (uint32_t)before;
    uint32_t out = g_before + min(e_before, (uint32_t)krem);   // ties before this thread are taken first
    int left_e = (int)min(ne, (uint32_t)max(0, krem - (int)e_before));
    // the key of column w * 32 + b is wbase + b (identity map, and block maps whose blocks are whole
    // bitmap words), else list[w * 32 + b] (list maps) or map_col (other block sizes)
    const int32_t* lrow = a.map.kind == kMapIdentity ? nullptr : a.map.list + (int64_t)rd.list * a.map.list_ld;
    const bool per_word = a.map.kind == kMapIdentity || (a.map.kind == kMapBlocks && (a.map.block & 31) == 0);
    for (int w = w0; w < w1; ++w) {
        uint32_t e = eqmap[w], te = 0;
        for (; left_e > 0 && e; --left_e) {   // the lowest remaining ties
            const uint32_t low = e & (0u - e);
            te |= low;
            e ^= low;
        }
        uint32_t bits = gtmap[w] | te;
        if (!bits) continue;
        const int c0 = w * 32;
        const int32_t wbase = a.map.kind == kMapIdentity ? c0 + a.map.offset
                              : per_word ? lrow[c0 / a.map.block] * a.map.block + c0 % a.map.block
                                         : 0;
        for (; bits; bits &= bits - 1) {
            const int b = __ffs(bits) - 1;
            const int col = c0 + b;
            const int32_t key = per_word ? wbase + b : a.map.kind == kMapList ? lrow[col] : map_col(a.map, rd, col);
            if (!DSA_CHECK(out < (uint32_t)k && key >= 0, a.status, 202)) { ++out; continue; }   // output slot, key
            if (staged) {   // the column: its score is read in the write-out, every thread's loads together
                stage[out] = key;
                if (osc) stage[k + out] = col;
            } else {
                oidx[out] = key;
                if (osc) osc[out] = key_score(score_key(__ldg(src + col)));
            }
            ++out;
        }
    }
    const int n_out = min(n, k);
    constexpr int kNaN = 0x7fc00000;
    if (!staged) {
        for (int j = n_out + tid; j < k; j += NT) {
            oidx[j] = -1;
            if (osc) osc[j] = __int_as_float(kNaN);
        }
        return;
    }
    __syncthreads();
    const bool vec = (k & 3) == 0 && ((reinterpret_cast<uintptr_t>(oidx) | reinterpret_cast<uintptr_t>(osc)) & 15) == 0;
    if (vec) {
        for (int j = 4 * tid; j < k; j += 4 * NT) {
            int4 v = *reinterpret_cast<const int4*>(stage + j);
            if (j + 3 >= n_out) {
                v.x = j < n_out ? v.x : -1;
                v.y = j + 1 < n_out ? v.y : -1;
                v.z = j + 2 < n_out ? v.z : -1;
                v.w = j + 3 < n_out ? v.w : -1;
            }
            *reinterpret_cast<int4*>(oidx + j) = v;
            if (osc) {
                const int4 c = *reinterpret_cast<const int4*>(stage + k + j);
                float4 f;
                f.x = j < n_out ? key_score(score_key(__ldg(src + c.x))) : __int_as_float(kNaN);
                f.y = j + 1 < n_out ? key_score(score_key(__ldg(src + c.y))) : __int_as_float(kNaN);
                f.z = j + 2 < n_out ? key_score(score_key(__ldg(src + c.z))) : __int_as_float(kNaN);
                f.w = j + 3 < n_out ? key_score(score_key(__ldg(src + c.w))) : __int_as_float(kNaN);
                *reinterpret_cast<float4*>(osc + j) = f;
            }
        }
    } else {
        for (int j = tid; j < k; j += NT) {
            oidx[j] = j < n_out ? stage[j] : -1;
            if (osc) osc[j] = j < n_out ? key_score(score_key(__ldg(src + stage[k + j]))) : __int_as_float(kNaN);
        }
    }
}

// One CTA per row: steps 1-4 above.
template <int NT>
__global__ void __launch_bounds__(NT, 1024 / NT) select_stream_kernel(SelectArgs a)
{
    extern __shared__ __align__(16) uint8_t sel_smem[];
    uint32_t* sample = reinterpret_cast<uint32_t*>(sel_smem);
    const int cap = a.buf_cap;
    uint64_t* buf = reinterpret_cast<uint64_t*>(sel_smem + a.sample_bytes);
    uint32_t* gtmap = reinterpret_cast<uint32_t*>(sel_smem + a.sample_bytes + (size_t)cap * 8);
    __shared__ SelScalars<NT> sh;
    grid_dep_wait();     // the scores come from the previous kernel
    grid_dep_launch();

    const int r = blockIdx.x;
    if (a.n_rows_dev && r >= *a.n_rows_dev) return;   // uniform exit
    const RowDesc rd = a.rows[r];
    const int n = rd.ncols;
    const int k = a.k;
    const float* src = a.S + (int64_t)(a.src_from_list ? rd.list : r) * a.ld_s;
    const int nwords = (n + 31) >> 5;
    uint32_t* eqmap = gtmap + nwords;
    if (n > k) prefetch_row_l2(src, n);

    for (int w = threadIdx.x; w < 2 * nwords; w += NT) gtmap[w] = 0;
    int krem = n;   // ties at T still to take (every column when n <= k)
    if (n > k) {
        const uint32_t tau =
            sel_threshold<NT>(src, n, k, cap, sample, sh, a.capped_sample ? capped_sample_size(n, k) : 0);
        if (threadIdx.x == 0) sh.count = 0;
        __syncthreads();
        sel_append<NT>(src, 0, n, tau, buf, cap, sh);
        __syncthreads();
        sel_mark<NT>(src, n, k, buf, (int)sh.count, cap, krem, gtmap, eqmap, sh, a.status);
    } else {
        __syncthreads();
        sel_mark_all<NT>(n, gtmap);
    }
    __syncthreads();
    sel_emit<NT>(a, rd, a.out_from_qrow ? rd.qrow : r, src, n, krem, gtmap, eqmap, reinterpret_cast<int32_t*>(sel_smem),
                 (a.sample_bytes + cap * 8) / 4, sh);
}

// Few long rows: P CTAs per row (blockIdx.x = r * P + p).  Every CTA of a row derives the same
// tau from the row's sample (step 1) and appends the candidates of its column chunk (step 2)
// to the row's global buffer gbuf[r * cap, (r + 1) * cap), counting them in ctr[2r]; the last
// CTA of the row to finish (ticket ctr[2r + 1]) ranks the buffer and writes the row (steps
// 3-4), then zeroes the row's two counters.  ctr must be zero at launch.
template <int NT>
__global__ void __launch_bounds__(NT, 1024 / NT) select_split_kernel(SelectArgs a, uint64_t* gbuf, uint32_t* ctr, int P)
{
    extern __shared__ __align__(16) uint8_t sel_smem[];
    uint32_t* sample = reinterpret_cast<uint32_t*>(sel_smem);
    const int cap = a.buf_cap;
    uint64_t* buf = reinterpret_cast<uint64_t*>(sel_smem + a.sample_bytes);
    uint32_t* gtmap = reinterpret_cast<uint32_t*>(sel_smem + a.sample_bytes + (size_t)cap * 8);
    __shared__ SelScalars<NT> sh;
    grid_dep_wait();     // the scores come from the previous kernel
    grid_dep_launch();

    const int r = blockIdx.x / P, p = blockIdx.x % P;
    const RowDesc rd = a.rows[r];
    const int n = rd.ncols;
    const int k = a.k;
    const float* src = a.S + (int64_t)(a.src_from_list ? rd.list : r) * a.ld_s;
    const int tid = threadIdx.x;
    uint64_t* g = gbuf + (int64_t)r * cap;

    if (n > k) {
        const int chunk = ((n + P - 1) / P + 127) & ~127;
        const int c0 = min(n, p * chunk), c1 = min(n, c0 + chunk);
        prefetch_row_l2(src + c0, c1 - c0);
        const uint32_t tau = sel_threshold<NT>(src, n, k, cap, sample, sh);
        if (tid == 0) sh.count = 0;
        __syncthreads();
        sel_append<NT>(src, c0, c1, tau, buf, cap, sh);
        __syncthreads();
        // the whole count goes into the row's total, so a chunk that overflowed its own buffer
        // also overflows the row's
        if (tid == 0) sh.base = sh.count > 0 ? atomicAdd(&ctr[2 * r], sh.count) : 0u;
        __syncthreads();
        const uint32_t base = sh.base, local = min(sh.count, (uint32_t)cap);
        for (uint32_t i = tid; i < local && base + i < (uint32_t)cap; i += NT) g[base + i] = buf[i];
        __threadfence();
    }
    __syncthreads();
    if (tid == 0) sh.last = atomicAdd(&ctr[2 * r + 1], 1u) == (uint32_t)(P - 1) ? 1u : 0u;
    __syncthreads();
    if (!sh.last) return;

    // ---- the row's last CTA: every other CTA's candidates are in g
    __threadfence();
    const int nwords = (n + 31) >> 5;
    uint32_t* eqmap = gtmap + nwords;
    for (int w = tid; w < 2 * nwords; w += NT) gtmap[w] = 0;
    if (tid == 0) {
        sh.count = *reinterpret_cast<volatile uint32_t*>(&ctr[2 * r]);
        ctr[2 * r] = 0u;       // ready for the next launch
        ctr[2 * r + 1] = 0u;
    }
    __syncthreads();
    int krem = n;
    if (n > k) {
        const int count = (int)sh.count;
        if (count >= k && count <= cap)
            for (int i = tid; i < count; i += NT) buf[i] = __ldcg(reinterpret_cast<const unsigned long long*>(g) + i);
        __syncthreads();
        sel_mark<NT>(src, n, k, buf, count, cap, krem, gtmap, eqmap, sh, a.status);
    } else {
        sel_mark_all<NT>(n, gtmap);
    }
    __syncthreads();
    sel_emit<NT>(a, rd, r, src, n, krem, gtmap, eqmap, reinterpret_cast<int32_t*>(sel_smem),
                 (a.sample_bytes + cap * 8) / 4, sh);
}

}  // namespace dsa
