// Exact per-row top-k for few long rows (decode): the P CTAs of a row form one thread-block
// cluster (2 <= P <= 8) and share the steps of select.cuh through distributed shared memory,
// instead of handing candidates to one finishing CTA through L2.
//
//   1. threshold: every CTA ranks the row's whole sample (the same m/32 runs of 32 columns
//      select_stream_kernel reads) by itself, the same way, so all find the same tau;
//   2. each CTA appends the columns of its chunk with key >= tau to its own candidate buffer;
//   3. the CTAs copy their candidates into the leader's buffer (offsets from one atomic on the
//      leader's counter); if the union holds >= k entries and nothing overflowed, the leader
//      ranks it (T and the number of T-ties to take), otherwise it ranks the whole row itself;
//   4. each CTA marks its own chunk (> T, == T) in its own bitmaps; the per-CTA counts go through
//      the leader; each CTA writes its chunk's columns at its offset, the T-ties taken in column
//      order across the chunks.
// Every cluster barrier is reached by every thread of every CTA, in the same order: the
// branches between barriers depend only on the row, which the whole cluster shares.
#pragma once

#include <cooperative_groups.h>

#include "select.cuh"

namespace dsa {

namespace cg = cooperative_groups;

constexpr int kClusterMaxParts = 8;

// The two halves of a cluster barrier: every thread of every CTA arrives (release), and a later
// wait (acquire) returns once all have arrived; the work between them overlaps the barrier.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// Scalars the row's CTAs exchange; the leader's copy is the one read.
struct alignas(16) ClusterShared {
    uint32_t gt[kClusterMaxParts];   // each CTA's marked counts (> T, == T)
    uint32_t eq[kClusterMaxParts];
    uint32_t count;                  // candidates in the leader's buffer
    uint32_t overflow;               // nonzero: some buffer overflowed
    uint32_t T;                      // the row's k-th key
    int32_t krem;                    // ties at T to take
    uint32_t mode;                   // 0: T from the candidates, 1: from the whole row, 2: every column
};

// Dynamic shared memory of select_cluster_kernel: the sample, the CTA's candidate buffer, the
// leader's union buffer (cap entries each) and two bitmaps of one chunk (chunk_words words each).
__host__ __device__ inline size_t cluster_smem_bytes(size_t sample_bytes, int cap, int chunk_words)
{
    return sample_bytes + (size_t)cap * 16 + (size_t)chunk_words * 8;
}

// Grid: P CTAs per row (blockIdx.x = row * P + cluster rank), launched as clusters of P.
// a.buf_cap: entries of each candidate buffer; chunk_words: bitmap words of the longest chunk.
template <int NT>
__global__ void __launch_bounds__(NT, 1) select_cluster_kernel(SelectArgs a, int P, int chunk_words)
{
    extern __shared__ __align__(16) uint8_t sel_smem[];
    const int cap = a.buf_cap;
    uint32_t* sample = reinterpret_cast<uint32_t*>(sel_smem);
    uint64_t* cand = reinterpret_cast<uint64_t*>(sel_smem + a.sample_bytes);
    uint64_t* gather = cand + cap;
    uint32_t* gtmap = reinterpret_cast<uint32_t*>(gather + cap);
    uint32_t* eqmap = gtmap + chunk_words;
    __shared__ SelScalars<NT> sh;
    __shared__ ClusterShared cs;
    cg::cluster_group cl = cg::this_cluster();
    const int p = (int)cl.block_rank();
    ClusterShared* lead = cl.map_shared_rank(&cs, 0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    grid_dep_wait();     // the scores come from the previous kernel
    grid_dep_launch();

    const int r = blockIdx.x / P;
    const RowDesc rd = a.rows[r];
    const int n = rd.ncols;
    const int k = a.k;
    const float* src = a.S + (int64_t)(a.src_from_list ? rd.list : r) * a.ld_s;
    const int chunk = ((n + P - 1) / P + 127) & ~127;
    const int c0 = min(n, p * chunk), c1 = min(n, c0 + chunk), nc = c1 - c0;
    const int words = (nc + 31) >> 5;
    if (n > k && nc > 0) prefetch_row_l2(src + c0, nc);
    for (int w = tid; w < 2 * chunk_words; w += NT) gtmap[w] = 0;   // both bitmaps
    if (tid == 0) {
        sh.count = 0;
        if (p == 0) {
            cs.count = 0;
            cs.overflow = 0;
        }
    }
    // the leader's counters are zero (and every CTA of the cluster runs) before any CTA touches the
    // leader's shared memory: arrive now, wait just before the first such access
    cluster_arrive();

    // ---- 1. tau: every CTA ranks the whole sample itself, the same way, so every CTA holds the same
    // tau with no cluster exchange (measured: the sample split among the CTAs, its digits summed in the
    // leader across two cluster barriers each, was 2-3.5 us slower per row)
    uint32_t tau = 0;
    if (n > k) tau = sel_threshold<NT>(src, n, k, cap, sample, sh, capped_sample_size(n, k));

    // ---- 2. this chunk's candidates; 3. into the leader's buffer
    if (n > k) sel_append<NT>(src, c0, c1, tau, cand, cap, sh);
    __syncthreads();
    cluster_wait();
    const uint32_t mine_c = sh.count;
    if (tid == 0) {
        uint32_t base = 0xffffffffu;
        if (n > k) {
            if (mine_c > (uint32_t)cap) atomicOr(&lead->overflow, 1u);
            else if (mine_c > 0) base = atomicAdd(&lead->count, mine_c);
        }
        sh.base = base;
    }
    __syncthreads();
    const uint32_t base = sh.base;
    if (base != 0xffffffffu) {
        if (base + mine_c <= (uint32_t)cap) {
            uint64_t* g = cl.map_shared_rank(gather, 0);
            for (uint32_t i = tid; i < mine_c; i += NT) g[base + i] = cand[i];
        } else if (tid == 0) {
            atomicOr(&lead->overflow, 1u);
        }
    }
    cl.sync();   // the union is in the leader

    // ---- the leader ranks the union (or the whole row)
    if (p == 0) {
        int krem = n;
        uint32_t T = 0u, mode = 2u;   // rows of at most k columns: every column
        if (n > k) {
            const int count = (int)cs.count;
            krem = k;
            if (!cs.overflow && count >= k && count <= cap) {
                uint32_t lo, hi;
                sel_buf_keys<NT>(gather, count, lo, hi, sh);
                T = radix_select_in<NT>([&](int i) { return (uint32_t)(gather[i] >> 32); }, count, krem, lo, hi,
                                        sh.hist, sh.scratch);
                mode = 0u;
            } else {
                T = radix_select<NT>([&](int i) { return score_key(__ldg(src + i)); }, n, krem, sh.hist,
                                     sh.scratch);
                mode = 1u;
            }
        }
        if (tid == 0) {
            cs.T = T;
            cs.krem = krem;
            cs.mode = mode;
        }
    }
    cl.sync();   // T, krem and the mode are in the leader

    // ---- 4. this chunk's marks
    const uint32_t T = lead->T;
    const int krem = lead->krem;
    const uint32_t mode = lead->mode;
    if (mode == 2u) {
        for (int w = tid; w < words; w += NT) gtmap[w] = (w + 1) * 32 <= nc ? 0xffffffffu : ((1u << (nc & 31)) - 1u);
    } else if (mode == 0u) {
        for (uint32_t i = tid; i < mine_c; i += NT) {   // every key >= T of the chunk is a candidate here
            const uint64_t e = cand[i];
            const uint32_t u = score_key(__uint_as_float((uint32_t)(e >> 32)));
            const uint32_t c = (uint32_t)e - (uint32_t)c0;
            if (!DSA_CHECK(c < (uint32_t)nc, a.status, 301)) continue;   // a column of this CTA's chunk
            if (u > T) atomicOr(&gtmap[c >> 5], 1u << (c & 31));
            else if (u == T) atomicOr(&eqmap[c >> 5], 1u << (c & 31));
        }
    } else {
        for (int c = tid; c < nc; c += NT) {
            const uint32_t u = score_key(__ldg(src + c0 + c));
            if (u > T) atomicOr(&gtmap[c >> 5], 1u << (c & 31));
            else if (u == T) atomicOr(&eqmap[c >> 5], 1u << (c & 31));
        }
    }
    __syncthreads();
    // thread-contiguous bitmap words; one block scan of the (> T, == T) counts
    const int wpt = (words + NT - 1) / NT;
    const int w0 = min(words, tid * wpt), w1 = min(words, w0 + wpt);
    uint32_t ng = 0, ne = 0;
    for (int w = w0; w < w1; ++w) {
        ng += __popc(gtmap[w]);
        ne += __popc(eqmap[w]);
    }
    const uint64_t own = ((uint64_t)ng << 32) | ne;
    uint64_t incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    uint64_t* wsum = reinterpret_cast<uint64_t*>(sh.hist);   // NT / 32 <= 32 entries
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    uint64_t before = incl - own, total = 0;
    for (int w = 0; w < NT / 32; ++w) {
        if (w < warp) before += wsum[w];
        total += wsum[w];
    }
    const uint32_t G = (uint32_t)(total >> 32), E = (uint32_t)total;   // this chunk's > T and == T
    if (tid == 0) {
        lead->gt[p] = G;
        lead->eq[p] = E;
    }
    cl.sync();   // every CTA's counts are in the leader
    // this chunk's first output and its share of the T-ties (ties go to the lowest columns, so
    // to the earlier chunks first)
    uint32_t out0 = 0, ties_before = 0;
    for (int q = 0; q < p; ++q) {
        const uint32_t eq_q = lead->eq[q];
        out0 += lead->gt[q] + min(eq_q, (uint32_t)max(0, krem - (int)ties_before));
        ties_before += eq_q;
    }
    const uint32_t quota = min(E, (uint32_t)max(0, krem - (int)ties_before));
    cluster_arrive();   // this CTA reads the leader's shared memory no more; the wait is at the end

    // ---- this chunk's columns, at out0 + (earlier threads' columns)
    int32_t* oidx = a.out_idx + (int64_t)r * a.ld_idx;
    float* osc = a.out_score ? a.out_score + (int64_t)r * a.ld_score : nullptr;
    const int cnt = (int)(G + quota);
    int32_t* stage = reinterpret_cast<int32_t*>(sel_smem);   // the sample and candidate buffer are free
    const bool staged = (osc ? 2 * cnt : cnt) <= (a.sample_bytes + cap * 8) / 4;
    const uint32_t g_before = (uint32_t)(before >> 32), e_before = (uint32_t)before;
    uint32_t out = g_before + min(e_before, quota);
    int left_e = (int)min(ne, (uint32_t)max(0, (int)quota - (int)e_before));
    const int32_t* lrow = a.map.kind == kMapIdentity ? nullptr : a.map.list + (int64_t)rd.list * a.map.list_ld;
    const bool per_word = a.map.kind == kMapIdentity || (a.map.kind == kMapBlocks && (a.map.block & 31) == 0);
    __syncthreads();   // the candidates were read (marks) before the stage overwrites them
    for (int w = w0; w < w1; ++w) {
        uint32_t e = eqmap[w], te = 0;
        for (; left_e > 0 && e; --left_e) {
            const uint32_t low = e & (0u - e);
            te |= low;
            e ^= low;
        }
        uint32_t bits = gtmap[w] | te;
        if (!bits) continue;
        const int cw = c0 + w * 32;   // c0 is a multiple of 128
        const int32_t wbase = a.map.kind == kMapIdentity ? cw + a.map.offset
                              : per_word ? lrow[cw / a.map.block] * a.map.block + cw % a.map.block
                                         : 0;
        for (; bits; bits &= bits - 1) {
            const int b = __ffs(bits) - 1;
            const int col = cw + b;
            const int32_t key = per_word ? wbase + b : a.map.kind == kMapList ? lrow[col] : map_col(a.map, rd, col);
            if (!DSA_CHECK(out0 + out < (uint32_t)k && out < (uint32_t)cnt && key >= 0, a.status, 302)) {
                ++out;
                continue;
            }
            if (staged) {   // the column: its score is read in the write-out, every thread's loads together
                stage[out] = key;
                if (osc) stage[cnt + out] = col;
            } else {
                oidx[out0 + out] = key;
                if (osc) osc[out0 + out] = key_score(score_key(__ldg(src + col)));
            }
            ++out;
        }
    }
    if (staged) {
        __syncthreads();
        for (int j = tid; j < cnt; j += NT) {
            oidx[out0 + j] = stage[j];
            if (osc) osc[out0 + j] = key_score(score_key(__ldg(src + stage[cnt + j])));
        }
    }
    if (p == 0) {   // padding past the row's columns
        for (int j = min(n, k) + tid; j < k; j += NT) {
            oidx[j] = -1;
            if (osc) osc[j] = __int_as_float(0x7fc00000);
        }
    }
    cluster_wait();   // the leader's shared memory outlives every read of it
}

}  // namespace dsa
