// Tensor-core (tcgen05 / TMEM) scoring of query rows against contiguous key
// tiles: the dense contraction of the lightning indexer with its epilogue.
//
// Orientation.  A key tile of 128 keys is the MMA's A operand (M = 128, one
// key per TMEM lane); the query-head pairs of up to 256 / H queries are the B
// operand (N = queries * H <= 256); K = d.  The fp32 accumulator row of a
// TMEM lane therefore holds q[t,h] . k[s] for one key s and every (t, h) of
// the tile, so each epilogue thread owns one key and reduces
// I[t,s] = sum_h w[t,h] * max(0, q[t,h] . k[s]) in registers with no
// cross-thread traffic.
//
// A CTA owns one work unit: up to 2 * (256 / H) consecutive queries of one
// segment (rows sharing one ordered set of candidate keys: a sequence's
// prefix, a PIVOT group's candidates, a HISA query's kept blocks) — two
// accumulators of 256 TMEM columns each, so every key tile in shared memory
// feeds two MMAs — and a range of its key tiles.  Column c of the segment is
// key map(c): contiguous key tiles are loaded with TMA tile loads, gathered
// ones with TMA gather4 (four rows per instruction and lane).  A warp issues
// its lanes' gather4 one after another, so a gathered tile (32 * d/64 of them)
// is split over three producer warps, each with its own full barrier.
// Roles:
//   warp 0      TMA producer: the query tile once, then a ring of key tiles
//   warp 1      TMEM allocator and MMA issuer (one thread)
//   warps 2..9  epilogue: TMEM -> registers, ReLU, weighted head sum, causal
//               mask, fp32 score store
//   warps 10-11 more producers of gathered tiles (idle for contiguous ones)
// The two accumulators are handed back and forth between MMA and epilogue
// with mbarriers, so the MMAs into one overlap the epilogue of the other.
// Keys kept in fp32 (HISA's pooled block keys) are scored as three bf16 planes:
// each value v is hi + mid + lo exactly (each part the leading 8 significant
// bits of what remains), the three tiles of a key tile pass through the ring
// one after another and accumulate into the same TMEM columns, so the sum
// q . hi + q . mid + q . lo is the fp32 dot product up to accumulation order.
// Every wait is bounded (1 s); a wait that runs out records an error in the
// workspace status word and the CTA drains its copies and MMAs and exits.
// A dense launch of one wave (decode) may do its own set-up (su.n_units > 0):
// each CTA computes its unit from the layout, the first split of each query
// tile writes the tile's rows for the select, CTA 0 clears the workspace
// header, and the epilogue takes the eligible counts from the positions; the
// call then needs no set-up kernel before it.
#pragma once

#include "ptx.cuh"
#include "setup.cuh"

namespace dsa {

constexpr int kTcProducers = 3;   // warps issuing gathered tiles: 0, 10, 11
constexpr int kTcThreads = 384;   // launches of contiguous tiles use the first 320 (warps 0..9)
constexpr int kTcThreadsTiles = 320;
constexpr int kTcMaxStages = 8;
constexpr uint32_t kErrSmemAlign = 3;

struct TcArgs {
    const TcUnit* units;
    const RowDesc* rows;
    ColMap map;              // column -> key index; identity: contiguous key tiles (TMA tile loads),
                             // otherwise each tile's 128 keys are gathered (TMA gather4)
    int32_t gather;          // 0: contiguous tiles, 1: gathered rows
    int32_t keep_keys;       // 1: other units read the same keys again: load them L2 evict-last
    const float* W;          // row rd.qrow: [H]
    float* S;                // score of launch row r, key s at S[r * ld_s + s]
    int64_t ld_s;
    uint32_t* status;
    int32_t n_stages;
    int32_t planes;          // 1, or 3: a key tile is the sum of three bf16 tiles (hi, mid, lo) plane_rows apart
    int64_t n_keys;          // rows of K (checked builds verify every gathered key row against it)
    int64_t plane_rows;
    int32_t block_tiles;     // contiguous launches: column c is key list[c / block] * block + c % block, with
                             // whole 128-key tiles per block (block a multiple of 128): one tile load each
    int32_t pad2_;
};

template <int D, int H>
struct TcShape {
    static constexpr int NQA = 256 / H;                  // queries per accumulator
    static constexpr int ROWB = D * 2 >= 128 ? 128 : 64;   // swizzle width = bytes of one box row
    static constexpr int BOXC = ROWB / 2;                 // bf16 elements per box row
    static constexpr int NBOX = D / BOXC;                 // boxes across d
    static constexpr int KSTEPS = D / 16;                 // MMAs of K = 16 per tile
    static constexpr uint32_t QBOX = 256u * ROWB;         // one Q box: 256 rows
    static constexpr uint32_t QACC = 256u * D * 2;        // Q operand of one accumulator
    static constexpr uint32_t KBOX = 128u * ROWB;
    static constexpr uint32_t KTILE = 128u * D * 2;
    static constexpr uint32_t W_BYTES = 2u * NQA * H * 4;
    static constexpr uint32_t NC_BYTES = 2u * NQA * 4;
    static constexpr uint32_t BAR_BYTES = 512;

    // Q tiles, key stages, W, eligible counts; the barriers and TMEM slot sit in the last
    // BAR_BYTES of the allocation, a place the prologue knows before the unit is read.
    __host__ __device__ static uint32_t smem_bytes(int n_acc, int n_stages)
    {
        return n_acc * QACC + n_stages * KTILE + W_BYTES + NC_BYTES + BAR_BYTES;
    }
};

__device__ __forceinline__ uint32_t dynamic_smem_size()
{
    uint32_t x;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(x));
    return x;
}

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, uint32_t* status, uint32_t where,
                                        volatile int32_t* abort_flag)
{
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 256; ++i)
            if (mbar_test(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            record_error(status, kErrWaitTimeout, where);
            *abort_flag = 1;
            return false;
        }
    }
}

// MODE kTcTiles: contiguous key tiles; kTcGather: the unit's key tiles are gathered through the
// column map (a.gather == 1); kTcBlocks: contiguous tiles at computed rows, the three planes of
// fp32 keys (a.planes) or whole 128-key tiles of a block map (a.block_tiles).  The cases are
// compiled apart, so the dense scan keeps the leanest producer and MMA-issuer loops.
enum : int { kTcTiles = 0, kTcGather = 1, kTcBlocks = 2 };

template <int D, int H, int MODE>
__global__ void __launch_bounds__(MODE == kTcGather ? kTcThreads : kTcThreadsTiles, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmKg, TcArgs a, const __grid_constant__ DenseSetupArgs su)
{
    constexpr bool GATHER = MODE == kTcGather;
    constexpr bool EXT = MODE == kTcBlocks;
    using SH = TcShape<D, H>;
    constexpr int NP = GATHER ? kTcProducers : 1;   // producers with a full barrier per stage
    constexpr int NQA = SH::NQA;
    constexpr int QH = NQA / 2;   // queries of one accumulator handled by one epilogue half

    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {   // the swizzled tiles need 1024-byte alignment (uniform exit)
        if (threadIdx.x == 0) record_error(a.status, kErrSmemAlign, blockIdx.x);
        return;
    }
    const int n_stages = a.n_stages;
    // full[p * n_stages + s]: producer p's part of stage s has landed
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + dynamic_smem_size() - SH::BAR_BYTES);
    uint64_t* empty = full + NP * n_stages;
    uint64_t* qfull = empty + n_stages;
    uint64_t* tfull = qfull + 1;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);

    // Prologue (may overlap the previous kernel): barriers, TMEM, descriptor prefetch.
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < n_stages; ++i) {
            for (int p = 0; p < NP; ++p) mbar_init(&full[p * n_stages + i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(qfull, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 8 * 32);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(GATHER ? &tmKg : &tmK);
    }
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    grid_dep_wait();     // the unit table and rows come from earlier kernels
    // (no early launch of the next kernel: its CTAs waiting on freed SMs slowed decode down)
    const bool own_setup = !GATHER && !EXT && su.n_units > 0;
    int seq_len = 0;     // own set-up: the unit's sequence length
    TcUnit u;
    if (own_setup) {
        int seq;
        u = dense_unit(su, blockIdx.x, seq, seq_len);
        if (blockIdx.x == 0)   // the call's status word and select counters start at zero
            for (int i = threadIdx.x; i < su.header_words; i += blockDim.x) su.header[i] = 0u;
        if ((int)blockIdx.x % su.splits == 0 && (int)threadIdx.x < u.nrows) {   // the tile's rows, for the select
            const int r = u.row0 + threadIdx.x;
            su.rows[r] = RowDesc{r, seq, eligible_count(su.q_pos[r], seq_len), 0};
        }
    } else {
        u = a.units[blockIdx.x];
    }
    const bool active = u.kt1 > u.kt0 && u.nrows > 0;   // uniform over the CTA
    const int n_acc = u.nrows > NQA ? 2 : 1;
    uint8_t* sQ = smem;
    uint8_t* sK = sQ + n_acc * SH::QACC;
    float* sW = reinterpret_cast<float*>(sK + n_stages * SH::KTILE);
    int32_t* sNc = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(sW) + SH::W_BYTES);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nkt = u.kt1 - u.kt0;

    if (!active) {
        // nothing to score: fall through to the TMEM release
    } else if (warp == 0 || (GATHER && warp >= 10)) {
        // ------------------------------------------------------ producers
        const int pw = warp == 0 ? 0 : warp - 9;   // producer index
        const int krow0 = u.krow0;
        if (pw == 0 && lane == 0) {
            mbar_arrive_expect_tx(qfull, n_acc * SH::QACC);
            for (int acc = 0; acc < n_acc; ++acc)
                for (int bx = 0; bx < SH::NBOX; ++bx)
                    tma_load_2d(sQ + acc * SH::QACC + bx * SH::QBOX, &tmQ, bx * SH::BOXC, (u.qrow + acc * NQA) * H,
                                qfull);
        }
        // Gathered tiles: item w = (box w / 32, rows 4 (w % 32) .. +3) of a tile goes to producer
        // w % kTcProducers, lane w / kTcProducers.
        constexpr int kItems = 32 * SH::NBOX;
        const int w = lane * kTcProducers + pw;
        const bool has_item = w < kItems;
        const int rg = w % 32, ibox = w / 32;
        const uint32_t my_bytes = (uint32_t)((kItems - pw + kTcProducers - 1) / kTcProducers) * 4 * SH::ROWB;
        uint64_t* my_full = full + pw * n_stages;
        // the columns of the unit that exist (tiles past them read column 0's key)
        int ncmax = 0, list = 0;
        if (GATHER || (EXT && a.block_tiles)) list = a.rows[u.row0].list;
        if (GATHER) {
            for (int j = lane; j < u.nrows; j += 32) ncmax = max(ncmax, a.rows[u.row0 + j].ncols);
            ncmax = __reduce_max_sync(0xffffffffu, ncmax);
        }
        const RowDesc first{0, 0, 0, list};   // map_col reads only the list row
        const int32_t* lrow = (GATHER || (EXT && a.block_tiles)) && a.map.kind != kMapIdentity
                                  ? a.map.list + (int64_t)list * a.map.list_ld : nullptr;
        const bool list4 = a.map.kind == kMapList && (reinterpret_cast<uintptr_t>(lrow) & 15) == 0;
        const bool block4 = a.map.kind == kMapBlocks && (a.map.block & 3) == 0;
        // Key rows of this lane's four rows (columns c0 .. c0+3) of tile i: one 16-byte list load,
        // or one block entry, when the four columns exist.
        auto tile_rows = [&](int i, int (&y)[4]) {
            const int c0 = (u.kt0 + i) * 128 + 4 * rg;
            if (c0 + 3 < ncmax && list4) {
                const int4 v = __ldg(reinterpret_cast<const int4*>(lrow + c0));
                y[0] = krow0 + v.x; y[1] = krow0 + v.y; y[2] = krow0 + v.z; y[3] = krow0 + v.w;
            } else if (c0 + 3 < ncmax && block4) {
                const int base = krow0 + __ldg(lrow + c0 / a.map.block) * a.map.block + c0 % a.map.block;
                y[0] = base; y[1] = base + 1; y[2] = base + 2; y[3] = base + 3;
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) y[e] = krow0 + map_col(a.map, first, c0 + e < ncmax ? c0 + e : 0);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e)   // a gathered key row of K (an out-of-range row would read zeros)
                if (!DSA_CHECK(y[e] >= 0 && y[e] < a.n_keys, a.status, 101)) y[e] = 0;
        };
        // Keys other units read again stay in L2 while the score rows stream out.
        const uint64_t keep_keys = l2_policy_evict_last();
        int ynext[4] = {0, 0, 0, 0};   // the next gathered tile's rows, loaded a tile ahead
        if (GATHER && has_item && nkt > 0) tile_rows(0, ynext);
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        const int planes = EXT ? a.planes : 1;
        int32_t blk = 0;   // block tiles: lane l holds the block of tile i0 + l
        for (int e = 0; e < nkt * planes; ++e) {
            const int i = EXT ? e / planes : e, pl = EXT ? e - i * planes : 0;
            int ok = 1;
            if (lane == 0) ok = tc_wait(&empty[stage], phase ^ 1u, a.status, 1, abort_flag) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            if constexpr (!GATHER) {
                int krow;
                if (EXT && a.block_tiles) {
                    if ((i & 31) == 0 && pl == 0) {   // the next 32 tiles' blocks, one load per lane
                        const int c = (u.kt0 + i + lane) * 128;
                        blk = i + lane < nkt ? __ldg(lrow + c / a.map.block) : 0;
                    }
                    const int c0 = (u.kt0 + i) * 128;
                    krow = krow0 + __shfl_sync(0xffffffffu, blk, i & 31) * a.map.block + c0 % a.map.block;
                    if (!DSA_CHECK(krow >= 0 && krow < a.n_keys, a.status, 102)) krow = 0;   // a block's first key row
                } else if (EXT) {
                    krow = krow0 + (u.kt0 + i) * 128 + (int)(pl * a.plane_rows);
                } else {
                    krow = krow0 + (u.kt0 + i) * 128;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&my_full[stage], SH::KTILE);
                    for (int bx = 0; bx < SH::NBOX; ++bx) {
                        if (a.keep_keys)
                            tma_load_2d_hint(sK + stage * SH::KTILE + bx * SH::KBOX, &tmK, bx * SH::BOXC, krow,
                                             &my_full[stage], keep_keys);
                        else
                            tma_load_2d(sK + stage * SH::KTILE + bx * SH::KBOX, &tmK, bx * SH::BOXC, krow,
                                        &my_full[stage]);
                    }
                }
            } else {
                if (lane == 0) mbar_arrive_expect_tx(&my_full[stage], my_bytes);
                __syncwarp();
                if (has_item) {
                    const int y[4] = {ynext[0], ynext[1], ynext[2], ynext[3]};
                    tma_gather4_2d_hint(sK + stage * SH::KTILE + ibox * SH::KBOX + 4 * rg * SH::ROWB, &tmKg,
                                        ibox * SH::BOXC, y[0], y[1], y[2], y[3], &my_full[stage], keep_keys);
                    if (i + 1 < nkt) tile_rows(i + 1, ynext);   // in flight while the next slot frees up
                }
            }
            ++issued;
            if (++stage == n_stages) { stage = 0; phase ^= 1u; }
        }
        // Before leaving, every copy this warp started must have landed.
        if (lane == 0 && *abort_flag) {
            if (pw == 0) mbar_wait(qfull, 0, a.status, 10);
            for (int back = 1; back <= n_stages && back <= issued; ++back) {
                const int i = issued - back;
                mbar_wait(&my_full[i % n_stages], (uint32_t)((i / n_stages) & 1), a.status, 11);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t idesc[2];
            for (int acc = 0; acc < 2; ++acc) {
                int nq = u.nrows - acc * NQA;
                nq = nq < NQA ? nq : NQA;
                int N = ((nq > 0 ? nq : 1) * H + 15) & ~15;
                idesc[acc] = idesc_bf16_f32(128, N);
            }
            if (tc_wait(qfull, 0, a.status, 2, abort_flag)) {
                tc_fence_after();
                int stage = 0;
                uint32_t phase = 0;
                uint32_t tph[2] = {0, 0};
                const int planes = EXT ? a.planes : 1;
                for (int e = 0; e < nkt * planes && !*abort_flag; ++e) {
                    const int i = EXT ? e / planes : e, pl = EXT ? e - i * planes : 0;
                    bool landed = true;
                    for (int p = 0; p < NP && landed; ++p)
                        landed = tc_wait(&full[p * n_stages + stage], phase, a.status, 3, abort_flag);
                    if (!landed) break;
                    tc_fence_after();
                    for (int qb = 0; qb < n_acc; ++qb) {
                        // one query block: the two accumulators alternate tile by tile
                        const int slot = n_acc == 1 ? (i & 1) : qb;
                        if (pl == 0) {   // a tile's first plane starts the accumulator afresh
                            if (!tc_wait(&tempty[slot], tph[slot] ^ 1u, a.status, 4, abort_flag)) break;
                            tc_fence_after();
                        }
                        const uint32_t d = tmem + slot * 256;
#pragma unroll
                        for (int kk = 0; kk < SH::KSTEPS; ++kk) {
                            const int bx = kk / (SH::BOXC / 16);
                            const uint32_t ko = (kk % (SH::BOXC / 16)) * 32;
                            const uint64_t ad =
                                smem_desc_kmajor(smem_u32(sK + stage * SH::KTILE + bx * SH::KBOX) + ko, SH::ROWB);
                            const uint64_t bd =
                                smem_desc_kmajor(smem_u32(sQ + qb * SH::QACC + bx * SH::QBOX) + ko, SH::ROWB);
                            tc_mma(d, ad, bd, idesc[qb], kk > 0 || pl > 0 ? 1u : 0u);
                        }
                        if (pl == planes - 1) {
                            tc_commit(&tfull[slot]);
                            tph[slot] ^= 1u;
                        }
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == n_stages) { stage = 0; phase ^= 1u; }
                }
            }
            // All MMAs issued by this thread complete before TMEM is released.
            tc_commit(drain);
            mbar_wait(drain, 0, a.status, 12);
        }
        __syncwarp();
    } else {   // warps 2..9
        // ---------------------------------------------------------- epilogue
        // the tile's head weights and eligible counts, shared by the 8 epilogue warps
        for (int i = threadIdx.x - 64; i < 2 * NQA * H; i += 256) {
            const int j = i / H;
            const int qrow = own_setup ? u.row0 + j : j < u.nrows ? a.rows[u.row0 + j].qrow : 0;
            sW[i] = j < u.nrows ? a.W[(int64_t)qrow * H + (i % H)] : 0.f;
        }
        for (int j = threadIdx.x - 64; j < 2 * NQA; j += 256)
            sNc[j] = j >= u.nrows ? 0 : own_setup ? eligible_count(su.q_pos[u.row0 + j], seq_len) : a.rows[u.row0 + j].ncols;
        asm volatile("bar.sync 1, 256;" ::: "memory");   // named barrier of the epilogue warps only
        const int quarter = warp & 3;           // TMEM lanes this warp may read
        const int half = (warp - 2) >> 2;       // which 128 columns of an accumulator
        uint32_t tph[2] = {0, 0};
        for (int i = 0; i < nkt; ++i) {
            const int key = (u.kt0 + i) * 128 + quarter * 32 + lane;
            for (int acc = 0; acc < n_acc; ++acc) {   // acc: query block
                const int slot = n_acc == 1 ? (i & 1) : acc;
                if (!tc_wait(&tfull[slot], tph[slot], a.status, 5, abort_flag)) break;
                tph[slot] ^= 1u;
                tc_fence_after();
                float v[128];
                const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + slot * 256 + half * 128;
                tmem_ld32(taddr, v);
                tmem_ld32(taddr + 32, v + 32);
                tmem_ld32(taddr + 64, v + 64);
                tmem_ld32(taddr + 96, v + 96);
                tmem_ld_wait();
                tmem_regs_ready<128>(v);
                tc_fence_before();
                mbar_arrive(&tempty[slot]);   // the accumulator may be overwritten from here on

                const int jbase = acc * NQA + half * QH;
#pragma unroll
                for (int q = 0; q < QH; ++q) {
                    const int j = jbase + q;
                    const float* w = sW + j * H;
                    float s0 = 0.f, s1 = 0.f;
                    if constexpr (H % 4 == 0) {
                        // even heads into s0, odd into s1, as one packed pair: each fma.rn.f32x2 does two
                        // IEEE fp32 fmas, the same ones in the same order as two scalar chains
                        uint64_t acc = 0;   // (s0, s1) = (+0, +0)
#pragma unroll
                        for (int h = 0; h < H; h += 4) {
                            const float4 w4 = *reinterpret_cast<const float4*>(w + h);
                            acc = fma_f32x2(pack_f32x2(w4.x, w4.y),
                                            pack_f32x2(fmaxf(v[q * H + h], 0.f), fmaxf(v[q * H + h + 1], 0.f)), acc);
                            acc = fma_f32x2(pack_f32x2(w4.z, w4.w),
                                            pack_f32x2(fmaxf(v[q * H + h + 2], 0.f), fmaxf(v[q * H + h + 3], 0.f)), acc);
                        }
                        unpack_f32x2(acc, s0, s1);
                    } else {
#pragma unroll
                        for (int h = 0; h < H; ++h) s0 = fmaf(w[h], fmaxf(v[q * H + h], 0.f), s0);
                    }
                    if (j < u.nrows && key < sNc[j])   // streaming store: score rows are read once, later
                        __stcs(&a.S[(int64_t)(u.row0 + j) * a.ld_s + key], (s0 + s1) + 0.f);   // -0 -> +0
                }
            }
            if (*abort_flag) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace dsa
