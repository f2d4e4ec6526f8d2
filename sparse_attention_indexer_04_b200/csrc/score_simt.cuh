// CUDA-core scoring of rows against (mapped) key columns, fp32 FMA.
//
// Used where the operand is not a bf16 tensor-core tile: HISA's pooled fp32
// block keys.  A CTA scores one row against kSimtCols consecutive columns,
// four lanes (a quad) per two columns: lane j of the quad holds the
// 4-dimension groups j, j+4, j+8, ... of both columns' keys in registers (so
// a quad's loads of q_h read 64 consecutive bytes, and each feeds both
// columns), computes the partial dot products of every head over them, and
// two xor shuffles give every lane of the quad the head's full q_h . k; then
// I = sum_h w_h * max(0, q_h . k), in fp32.  Splitting the dimensions (not
// the heads) keeps one read of each key and a quarter of its registers per
// lane, so an SM holds enough warps to hide the FMA and shared-memory
// latencies of this short, latency-bound launch; the shared-memory reads of
// q are its limit, hence two columns per quad.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kSimtColsPerQuad = 2;           // columns per quad: each q load feeds both
constexpr int kSimtThreads = 256;
constexpr int kSimtCols = kSimtThreads / 4 * kSimtColsPerQuad;   // columns per CTA

struct ScoreArgs {
    const RowDesc* rows;
    int32_t n_rows;
    int32_t H;
    ColMap map;
    const __nv_bfloat16* Q;   // row rd.qrow: [H, D]
    const float* W;           // row rd.qrow: [H]
    const void* K;            // key rows, bf16 or fp32
    const int32_t* k_base;    // key row of (seq, key) = k_base[seq] + key
    float* S;                 // row r at S + r * ld_s
    int64_t ld_s;
    int32_t fill;             // columns [ncols, fill) receive -inf (0: none)
    int32_t pad_;
};

// The 4-dimension groups part, part + 4, part + 8, ... of a key row of D elements (bf16 or fp32) into
// registers: D / 4 values.
template <int D>
__device__ __forceinline__ void load_key_part(const __nv_bfloat16* kp, int part, float* kr)
{
    const uint2* p = reinterpret_cast<const uint2*>(kp);   // 4 bf16 per 8 bytes
#pragma unroll
    for (int m = 0; m < D / 16; ++m) {
        const uint2 v = __ldg(p + 4 * m + part);
        kr[4 * m] = __uint_as_float(v.x << 16);
        kr[4 * m + 1] = __uint_as_float(v.x & 0xffff0000u);
        kr[4 * m + 2] = __uint_as_float(v.y << 16);
        kr[4 * m + 3] = __uint_as_float(v.y & 0xffff0000u);
    }
}

template <int D>
__device__ __forceinline__ void load_key_part(const float* kp, int part, float* kr)
{
    const float4* p = reinterpret_cast<const float4*>(kp);
#pragma unroll
    for (int m = 0; m < D / 16; ++m) {
        const float4 v = __ldg(p + 4 * m + part);
        kr[4 * m] = v.x; kr[4 * m + 1] = v.y; kr[4 * m + 2] = v.z; kr[4 * m + 3] = v.w;
    }
}

template <int D, typename KT>
__global__ void __launch_bounds__(kSimtThreads) score_simt_kernel(ScoreArgs a)
{
    constexpr int DQ = D / 4;   // dimensions per lane
    static_assert(D % 16 == 0, "4-dimension groups, four per quad");
    extern __shared__ float sm[];
    const int r = blockIdx.x;
    const RowDesc rd = a.rows[r];
    const int col0 = blockIdx.y * kSimtCols;
    const int lim = max(rd.ncols, a.fill);
    if (col0 >= lim) return;
    float* sq = sm;
    float* sw = sm + a.H * D;
    // the row's query (H x D bf16, 16-byte loads, all of a thread's in flight at once) and weights
    const uint4* q = reinterpret_cast<const uint4*>(a.Q + (int64_t)rd.qrow * a.H * D);
    const int n8 = a.H * D / 8;
    constexpr int kPer = 64 * 128 / 8 / kSimtThreads;   // loads per thread for the largest query
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int i = threadIdx.x + u * kSimtThreads;
        if (i < n8) {
            const uint4 v = __ldg(q + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sq[8 * i + 2 * e] = __uint_as_float(w[e] << 16);
                sq[8 * i + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
            }
        }
    }
    for (int h = threadIdx.x; h < a.H; h += kSimtThreads) sw[h] = a.W[(int64_t)rd.qrow * a.H + h];
    __syncthreads();
    const int part = threadIdx.x & 3;   // which 4-dimension groups
    constexpr int C = kSimtColsPerQuad;
    const int colq = col0 + (threadIdx.x >> 2) * C;   // the quad's first column
    float kr[C][DQ];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        if (colq + c < rd.ncols) {
            const int32_t key = map_col(a.map, rd, colq + c);
            const KT* kp = reinterpret_cast<const KT*>(a.K) + (int64_t)(a.k_base[rd.seq] + key) * D;
            load_key_part<D>(kp, part, kr[c]);
        } else {
#pragma unroll
            for (int i = 0; i < DQ; ++i) kr[c][i] = 0.f;
        }
    }
    float acc[C];
#pragma unroll
    for (int c = 0; c < C; ++c) acc[c] = 0.f;
#pragma unroll 2
    for (int h = 0; h < a.H; ++h) {
        const float4* qh = reinterpret_cast<const float4*>(sq + h * D) + part;
        float d0[C], d1[C];
#pragma unroll
        for (int c = 0; c < C; ++c) { d0[c] = 0.f; d1[c] = 0.f; }
#pragma unroll
        for (int i = 0; i < DQ / 4; ++i) {
            const float4 qv = qh[4 * i];   // dimensions 4 (4 i + part) .. +3
#pragma unroll
            for (int c = 0; c < C; ++c) {
                d0[c] = fmaf(qv.x, kr[c][4 * i], d0[c]);
                d1[c] = fmaf(qv.y, kr[c][4 * i + 1], d1[c]);
                d0[c] = fmaf(qv.z, kr[c][4 * i + 2], d0[c]);
                d1[c] = fmaf(qv.w, kr[c][4 * i + 3], d1[c]);
            }
        }
        const float w = sw[h];
#pragma unroll
        for (int c = 0; c < C; ++c) {
            float dot = d0[c] + d1[c];
            dot += __shfl_xor_sync(0xffffffffu, dot, 1);   // the quad's four parts
            dot += __shfl_xor_sync(0xffffffffu, dot, 2);
            acc[c] = fmaf(w, fmaxf(dot, 0.f), acc[c]);
        }
    }
    if (part < C) {   // lane c of the quad writes column c
        float v = acc[0];
#pragma unroll
        for (int c = 1; c < C; ++c) v = part == c ? acc[c] : v;
        const int col = colq + part;
        if (col < lim) a.S[(int64_t)r * a.ld_s + col] = col < rd.ncols ? v + 0.f : -INFINITY;   // -0 -> +0
    }
}

}  // namespace dsa
