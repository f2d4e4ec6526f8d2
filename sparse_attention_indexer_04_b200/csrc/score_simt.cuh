// CUDA-core scoring of rows against (mapped) key columns, fp32 FMA.
//
// Used where the operand is not a bf16 tensor-core tile: HISA's pooled fp32
// block keys, and small or irregular rows.  One CTA scores one row against
// 128 consecutive columns; thread c holds its key in registers and walks
// the row's H heads, I = sum_h w_h * max(0, q_h . k), each dot product
// accumulated in fp32 as four interleaved partial sums (four independent
// FMA chains instead of one 128-long chain).
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kSimtCols = 128;

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

template <int D>
__device__ __forceinline__ void load_key(const __nv_bfloat16* kp, float* kr)
{
    const uint4* p = reinterpret_cast<const uint4*>(kp);
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        const uint4 v = __ldg(p + j);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            kr[8 * j + 2 * e] = __uint_as_float(w[e] << 16);
            kr[8 * j + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
        }
    }
}

template <int D>
__device__ __forceinline__ void load_key(const float* kp, float* kr)
{
    const float4* p = reinterpret_cast<const float4*>(kp);
#pragma unroll
    for (int j = 0; j < D / 4; ++j) {
        const float4 v = __ldg(p + j);
        kr[4 * j] = v.x; kr[4 * j + 1] = v.y; kr[4 * j + 2] = v.z; kr[4 * j + 3] = v.w;
    }
}

template <int D, typename KT>
__global__ void __launch_bounds__(kSimtCols) score_simt_kernel(ScoreArgs a)
{
    extern __shared__ float sm[];
    const int r = blockIdx.x;
    const RowDesc rd = a.rows[r];
    const int col0 = blockIdx.y * kSimtCols;
    const int lim = max(rd.ncols, a.fill);
    if (col0 >= lim) return;
    float* sq = sm;
    float* sw = sm + a.H * D;
    const __nv_bfloat16* q = a.Q + (int64_t)rd.qrow * a.H * D;
    for (int i = threadIdx.x; i < a.H * D; i += kSimtCols) sq[i] = __bfloat162float(q[i]);
    for (int h = threadIdx.x; h < a.H; h += kSimtCols) sw[h] = a.W[(int64_t)rd.qrow * a.H + h];
    __syncthreads();
    const int col = col0 + threadIdx.x;
    float out = -INFINITY;
    if (col < rd.ncols) {
        const int32_t key = map_col(a.map, rd, col);
        const KT* kp = reinterpret_cast<const KT*>(a.K) + (int64_t)(a.k_base[rd.seq] + key) * D;
        float kr[D];
        load_key<D>(kp, kr);
        float acc = 0.f;
#pragma unroll 2
        for (int h = 0; h < a.H; ++h) {
            const float4* qh = reinterpret_cast<const float4*>(sq + h * D);
            float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll
            for (int i = 0; i < D / 4; ++i) {
                const float4 qv = qh[i];
                d0 = fmaf(qv.x, kr[4 * i], d0);
                d1 = fmaf(qv.y, kr[4 * i + 1], d1);
                d2 = fmaf(qv.z, kr[4 * i + 2], d2);
                d3 = fmaf(qv.w, kr[4 * i + 3], d3);
            }
            acc = fmaf(sw[h], fmaxf((d0 + d1) + (d2 + d3), 0.f), acc);
        }
        out = acc + 0.f;   // -0 -> +0
    }
    if (col < lim) a.S[(int64_t)r * a.ld_s + col] = out;
}

}  // namespace dsa
