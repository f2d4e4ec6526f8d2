// libdsaidx C ABI: argument checks, workspace layout and kernel launches.
// Declarations and the contract of every entry point: include/dsa_index.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/dsa_index.h"
#include "common.cuh"
#include "score_simt.cuh"
#include "score_tc.cuh"
#include "select.cuh"
#include "select_cluster.cuh"
#include "select_regs.cuh"
#include "reuse.cuh"
#include "setup.cuh"

using namespace dsa;

namespace {

constexpr int32_t kMaxK = 16384;
constexpr int32_t kMaxCand = 16384;
// Bytes of materialised score rows per launch: 4 GiB holds a whole 32K prefill (one scoring launch
// of 4096 units and one select, through dense_topk_one_launch).  Measured on that prefill: 7.33 ms
// per step against 7.40 (2 GiB, two chunks) and 7.37-7.42 (1 GiB, four); 256 MiB (256 units, 1.7
// waves per launch) lost ~14 % to the last wave.
constexpr size_t kScoreBudget = size_t(4096) << 20;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace header: the status word (kStatusBytes), then two counters per row of the split-row
// select (kSplitMaxRows rows).  Each call clears the header once before its first launch.
constexpr int32_t kSplitMaxRows = 512;
constexpr size_t kHeaderBytes = kStatusBytes + size_t(kSplitMaxRows) * 2 * sizeof(uint32_t);

uint32_t* split_counters(void* ws) { return reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + kStatusBytes); }

// Sequential carve-out of a workspace; a dry run (base == nullptr) sizes it.
struct Carver {
    char* base;
    size_t off = kHeaderBytes;
    template <typename T>
    T* take(size_t count)
    {
        T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
        off = align256(off + count * sizeof(T));
        return p;
    }
};

bool head_dim_ok(int d) { return d == 32 || d == 64 || d == 128; }
bool heads_ok(int h) { return h >= 1 && h <= 64 && (h & (h - 1)) == 0; }

struct HostInfo {
    int32_t max_q = 0;   // longest query run of a sequence
    int32_t max_k = 0;   // longest key run of a sequence
};

dsa_status check_batch(const dsa_batch* b, HostInfo* info)
{
    if (!b) return DSA_ERR_INVALID_ARG;
    if (b->num_seqs < 1 || b->num_queries < 0 || b->num_keys < 0) return DSA_ERR_INVALID_ARG;
    if (!heads_ok(b->num_heads) || !head_dim_ok(b->head_dim)) return DSA_ERR_UNSUPPORTED;
    if (!b->q_offsets || !b->k_offsets || !b->q_offsets_host || !b->k_offsets_host)
        return DSA_ERR_INVALID_ARG;
    if (b->num_queries > 0 && !b->q_pos) return DSA_ERR_INVALID_ARG;
    const int32_t* qo = b->q_offsets_host;
    const int32_t* ko = b->k_offsets_host;
    if (qo[0] != 0 || ko[0] != 0) return DSA_ERR_INVALID_ARG;
    for (int i = 0; i < b->num_seqs; ++i) {
        if (qo[i + 1] < qo[i] || ko[i + 1] < ko[i]) return DSA_ERR_INVALID_ARG;
        info->max_q = std::max(info->max_q, qo[i + 1] - qo[i]);
        info->max_k = std::max(info->max_k, ko[i + 1] - ko[i]);
    }
    if (qo[b->num_seqs] != b->num_queries || ko[b->num_seqs] != b->num_keys) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

dsa_status check_tensors(const dsa_batch* b, const void* Q, const void* K, const float* W)
{
    if (b->num_queries > 0 && (!Q || !W)) return DSA_ERR_INVALID_ARG;
    if (b->num_keys > 0 && !K) return DSA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K)) & 15) return DSA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(W) & 3) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

dsa_status check_ws(void* ws, size_t ws_bytes, size_t need)
{
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255)) return DSA_ERR_WORKSPACE;
    return DSA_OK;
}

// The status word of the entry point running on this host thread: select launches hand it to their
// kernels (checked builds record index errors there).  Set by every entry point before its launches.
thread_local uint32_t* g_status = nullptr;

dsa_status launched()
{
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// Launches a kernel, with programmatic stream serialization when `pdl`: it may then be
// scheduled while the previous kernel on the stream still runs, and must call grid_dep_wait()
// before it touches memory an earlier kernel writes or reads.
template <typename... KArgs, typename... Args>
void launch_pdl(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                Args... args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    (void)cudaLaunchKernelEx(&cfg, kern, args...);   // errors surface through launched()
}

// Launches a kernel as clusters of `cluster` CTAs along x (with programmatic stream
// serialization, as launch_pdl).
template <typename... KArgs, typename... Args>
void launch_clustered(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, int cluster, cudaStream_t st,
                      Args... args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    (void)cudaLaunchKernelEx(&cfg, kern, args...);   // errors surface through launched()
}

// Programmatic launch pays off for the short kernels of decode (it hides each launch's latency
// behind the previous kernel) and cost the multi-wave prefill kernels ~4% when measured, so it
// is used when the grids involved fit in about two waves.
bool latency_bound(int64_t ctas) { return ctas <= 2 * 148; }

// ------------------------------------------------------------- profiling
// Kernel kinds timed by the optional profiler (dsa_profile_*).
enum ProfKind : int32_t {
    kProfSetup = 0, kProfScoreSimt, kProfSelect, kProfPool, kProfProxy, kProfScoreTc, kProfFill, kProfKinds
};
const char* const kProfNames[kProfKinds] = {"setup", "score_simt", "select_topk", "hisa_pool", "pivot_proxy",
                                            "score_tc", "fill"};

struct ProfRec {
    int32_t kind;
    cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
std::atomic<bool> g_prof_on{false};
std::vector<ProfRec> g_prof;
std::atomic<uint64_t> g_launches{0};

#define DSA_LAUNCH(kind, st, ...)      \
    do {                               \
        LaunchScope _ls((kind), (st)); \
        __VA_ARGS__;                   \
    } while (0)

// Counts one kernel launch; when profiling is on, brackets it with events on its stream.
struct LaunchScope {
    int32_t kind;
    cudaStream_t st;
    cudaEvent_t start = nullptr;
    LaunchScope(int32_t k, cudaStream_t s) : kind(k), st(s)
    {
        g_launches.fetch_add(1, std::memory_order_relaxed);
        if (g_prof_on.load(std::memory_order_relaxed) && cudaEventCreate(&start) == cudaSuccess)
            cudaEventRecord(start, st);
    }
    ~LaunchScope()
    {
        if (!start) return;
        cudaEvent_t stop;
        if (cudaEventCreate(&stop) != cudaSuccess) { cudaEventDestroy(start); return; }
        cudaEventRecord(stop, st);
        std::lock_guard<std::mutex> lk(g_prof_mu);
        g_prof.push_back(ProfRec{kind, start, stop});
    }
};

int64_t score_ld(int32_t cols) { return std::max<int64_t>(4, (cols + 3) & ~3); }

int32_t chunk_rows(int32_t n_rows, int64_t ld)
{
    const int64_t per = ld * int64_t(sizeof(float));
    return (int32_t)std::max<int64_t>(1, std::min<int64_t>(n_rows, int64_t(kScoreBudget) / per));
}

// ------------------------------------------------------------ launchers

template <typename KT>
dsa_status launch_score(const RowDesc* rows, int32_t n_rows, int32_t max_cols, const ColMap& map,
                        const void* Q, const float* W, int H, int D, const KT* K, const int32_t* k_base,
                        float* S, int64_t ld_s, int32_t fill, cudaStream_t st)
{
    if (n_rows <= 0) return DSA_OK;
    const int32_t cols = std::max(max_cols, fill);
    if (cols <= 0) return DSA_OK;
    ScoreArgs a{};
    a.rows = rows; a.n_rows = n_rows; a.H = H; a.map = map;
    a.Q = reinterpret_cast<const __nv_bfloat16*>(Q); a.W = W; a.K = K; a.k_base = k_base;
    a.S = S; a.ld_s = ld_s; a.fill = fill;
    const dim3 grid(n_rows, (cols + kSimtCols - 1) / kSimtCols);
    const size_t smem = size_t(H) * D * sizeof(float) + size_t(H) * sizeof(float);
    switch (D) {
    case 32: DSA_LAUNCH(kProfScoreSimt, st, score_simt_kernel<32, KT><<<grid, kSimtThreads, smem, st>>>(a)); break;
    case 64: DSA_LAUNCH(kProfScoreSimt, st, score_simt_kernel<64, KT><<<grid, kSimtThreads, smem, st>>>(a)); break;
    default: DSA_LAUNCH(kProfScoreSimt, st, score_simt_kernel<128, KT><<<grid, kSimtThreads, smem, st>>>(a)); break;
    }
    return launched();
}

// Dynamic shared memory the select kernels may take: a CTA's 227 KB less their static shared
// memory (SelScalars: the radix histogram and scalars, about 1.2 KB; 4 KB reserved).
constexpr size_t kSelectDynMax = (size_t)227 * 1024 - 4096;
static_assert(sizeof(SelScalars<512>) + 512 <= 4096, "select static shared memory");

// Threads per row of the streaming select: 256 when rows fill the GPU several times over, 512
// when there are few rows, k is large or the shared memory leaves at most two CTAs per SM (each
// row's phases are latency-bound), 1024 for k of 8192 or more (the candidate buffer then takes
// most of the shared memory: one CTA per SM).  Measured on the 32K prefill (32768 rows: 256 best),
// the 16 x 32K decode (32 rows: 512 best) and PIVOT's top-8192 candidate selection at 128K (1024:
// 3.12 ms against 3.44 with 512).
int select_threads(int32_t n_rows, int32_t k, size_t smem)
{
    return k >= 8192 ? 1024 : n_rows < 2 * 148 || k >= 4096 || smem > kSelectDynMax / 3 ? 512 : 256;
}

// Candidate buffer entries of the select: 1.75 k, or what fits in shared memory next to the
// bitmaps of max_cols columns (a smaller buffer only sends more rows down the full-row path).
int32_t select_cap(int32_t k, int32_t max_cols)
{
    const size_t fixed = select_smem_bytes(std::max(max_cols, 1), 0, k);
    const int fit = fixed < kSelectDynMax ? (int)((kSelectDynMax - fixed) / 8) & ~255 : 0;
    return std::max(256, std::min(select_buf_cap(k), fit));
}

// Whether rows of max_cols columns fit the select's shared memory (sample, a candidate buffer of
// at least 256 entries, two column bitmaps): up to 774,144 columns.
bool select_fits(int32_t k, int32_t max_cols)
{
    return select_smem_bytes(std::max(max_cols, 1), select_cap(k, max_cols), k) <= kSelectDynMax;
}

// Scratch of the split-row select: two counters per row in the workspace header (zero between
// launches) and a global candidate buffer of max_rows x select_cap entries.
struct SelectSplit {
    uint32_t* ctr = nullptr;
    uint64_t* buf = nullptr;
    int32_t max_rows = 0;
};

// Rows a plan may hand to the split select in one launch (0: never split).
int32_t split_rows_for(int32_t chunk) { return chunk <= 2 * 148 ? chunk : 0; }

// CTAs per row of the split select: one wave of at most 148 CTAs over all rows (more CTAs only
// lengthen the launch ramp; the per-row steps other than the scan do not shrink), each chunk at
// least 2048 columns (1 = use the one-CTA-per-row kernel).
int select_parts(int32_t n_rows, int32_t max_cols)
{
    if (n_rows <= 0) return 1;
    return std::max(1, std::min(148 / n_rows, max_cols / 2048));
}

template <typename Kern>
dsa_status set_smem(Kern kern, size_t smem)
{
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) == cudaSuccess
               ? DSA_OK
               : DSA_ERR_CUDA;
}

// The register top-k kernels, by row length (rows of at most 16,384 columns); smem: the staged
// output row.
template <template <int, int> class Launch, typename... Args>
dsa_status launch_regs(int32_t max_cols, size_t smem, Args&&... args)
{
    if (max_cols <= 2048) return Launch<256, 8>::run(smem, args...);
    if (max_cols <= 4096) return Launch<512, 8>::run(smem, args...);
    if (max_cols <= 8192) return Launch<1024, 8>::run(smem, args...);
    if (max_cols <= 12288) return Launch<1024, 12>::run(smem, args...);
    return Launch<1024, 16>::run(smem, args...);
}

template <int NT, int R>
struct RegsSelect {
    static dsa_status run(size_t smem, int32_t n_rows, const SelectArgs& a, cudaStream_t st)
    {
        dsa_status s = set_smem(select_regs_kernel<NT, R>, smem);
        if (s != DSA_OK) return s;
        DSA_LAUNCH(kProfSelect, st, launch_pdl(latency_bound(n_rows), select_regs_kernel<NT, R>, n_rows, NT, smem, st, a));
        return launched();
    }
};

// n_rows_dev (optional): only rows below the count a kernel wrote there are ranked, and each
// writes output row rows[r].qrow (the one-CTA-per-row kernel only).
dsa_status launch_select(const RowDesc* rows, int32_t n_rows, int32_t max_cols, int32_t k, const ColMap& map,
                         const float* S, int64_t ld_s, bool src_from_list, int32_t* out_idx, int64_t ld_idx,
                         float* out_score, int64_t ld_score, cudaStream_t st, const SelectSplit& sp = SelectSplit{},
                         const int32_t* n_rows_dev = nullptr)
{
    if (n_rows <= 0) return DSA_OK;
    SelectArgs a{};
    a.rows = rows; a.n_rows = n_rows; a.k = k; a.map = map; a.S = S; a.ld_s = ld_s;
    a.status = g_status;
    a.src_from_list = src_from_list ? 1 : 0;
    a.out_idx = out_idx; a.ld_idx = ld_idx; a.out_score = out_score; a.ld_score = ld_score;
    a.n_rows_dev = n_rows_dev;
    a.out_from_qrow = n_rows_dev ? 1 : 0;
    a.buf_cap = select_cap(k, max_cols);
    a.sample_bytes = (int32_t)select_sample_bytes(std::max(max_cols, 1), k);
    size_t smem = select_smem_bytes(std::max(max_cols, 1), a.buf_cap, k);
    const int m_cap = capped_sample_size(std::max(max_cols, 1), k);
    if (m_cap * 4 < a.sample_bytes && n_rows > 2 * 148) {
        // many long rows (PIVOT's group lists): a sample of at most 4096 columns and a candidate buffer
        // of 3k entries for the wider threshold, in the same shared memory (the ranking of the sample
        // is the one-CTA select's largest fixed cost per row)
        const size_t words = (size_t(std::max(max_cols, 1)) + 31) / 32;
        const int64_t fit = (int64_t(kSelectDynMax) - int64_t(m_cap) * 4 - int64_t(words) * 8) / 8;
        a.capped_sample = 1;
        a.sample_bytes = m_cap * 4;
        a.buf_cap = (int32_t)std::max<int64_t>(a.buf_cap, std::min<int64_t>((3 * int64_t(k) + 255) & ~255, fit & ~255));
        smem = size_t(a.sample_bytes) + size_t(a.buf_cap) * 8 + words * 8;
    }
    dsa_status s;
    const int P = select_parts(n_rows, max_cols);
    if (sp.buf && sp.ctr && n_rows <= sp.max_rows && P > 1 && !n_rows_dev) {
        // a row's CTAs as one cluster when they fit one (P <= 8), its shared memory layout fits and
        // the rows are long: measured, 16 x 128K 31-33 -> 27-28 us, 16 x 32K unchanged, and HISA's
        // ~8.4K-column token rows 3 us slower (ten cluster barriers against a short scan)
        const int chunk_words = ((((max_cols + P - 1) / P + 127) & ~127) + 31) / 32;
        // every CTA ranks the whole sample, so the cluster takes a smaller one (capped_sample_size)
        // and a candidate buffer of 3k entries for the wider threshold, as far as shared memory allows
        SelectArgs ca = a;
        ca.sample_bytes = capped_sample_size(std::max(max_cols, 1), k) * 4;
        const int64_t fit = (int64_t(kSelectDynMax) - ca.sample_bytes - int64_t(chunk_words) * 8) / 16;
        ca.buf_cap = (int32_t)std::max<int64_t>(a.buf_cap, std::min<int64_t>((3 * int64_t(k) + 255) & ~255, fit & ~255));
        const size_t csmem = cluster_smem_bytes(ca.sample_bytes, ca.buf_cap, chunk_words);
        if (P <= kClusterMaxParts && max_cols >= 16384 && csmem <= kSelectDynMax) {
            if ((s = set_smem(select_cluster_kernel<512>, csmem)) != DSA_OK) return s;
            DSA_LAUNCH(kProfSelect, st, launch_clustered(select_cluster_kernel<512>, n_rows * P, 512, csmem, P, st, ca,
                                                         P, chunk_words));
            return launched();
        }
        if ((s = set_smem(select_split_kernel<512>, smem)) != DSA_OK) return s;
        DSA_LAUNCH(kProfSelect, st, launch_pdl(true, select_split_kernel<512>, n_rows * P, 512, smem, st, a, sp.buf,
                                               sp.ctr, P));
        return launched();
    }
    switch (select_threads(n_rows, k, smem)) {
    case 1024:
        if ((s = set_smem(select_stream_kernel<1024>, smem)) != DSA_OK) return s;
        DSA_LAUNCH(kProfSelect, st, launch_pdl(latency_bound(n_rows), select_stream_kernel<1024>, n_rows, 1024, smem, st, a));
        break;
    case 512:
        if ((s = set_smem(select_stream_kernel<512>, smem)) != DSA_OK) return s;
        DSA_LAUNCH(kProfSelect, st, launch_pdl(latency_bound(n_rows), select_stream_kernel<512>, n_rows, 512, smem, st, a));
        break;
    default:
        if ((s = set_smem(select_stream_kernel<256>, smem)) != DSA_OK) return s;
        DSA_LAUNCH(kProfSelect, st, launch_pdl(latency_bound(n_rows), select_stream_kernel<256>, n_rows, 256, smem, st, a));
        break;
    }
    return launched();
}

// Score then select, in row chunks that fit the score buffer.
template <typename KT>
dsa_status score_and_select(const RowDesc* rows, int32_t n_rows, int32_t max_cols, const ColMap& map,
                            const void* Q, const float* W, int H, int D, const KT* K, const int32_t* k_base,
                            float* Sbuf, int32_t k, int32_t* idx, int64_t ld_idx, float* scores,
                            cudaStream_t st)
{
    const int64_t ld = score_ld(max_cols);
    const int32_t chunk = chunk_rows(n_rows, ld);
    for (int32_t r0 = 0; r0 < n_rows; r0 += chunk) {
        const int32_t nr = std::min(chunk, n_rows - r0);
        dsa_status s = launch_score<KT>(rows + r0, nr, max_cols, map, Q, W, H, D, K, k_base, Sbuf, ld, 0, st);
        if (s != DSA_OK) return s;
        s = launch_select(rows + r0, nr, max_cols, k, map, Sbuf, ld, false, idx + int64_t(r0) * ld_idx, ld_idx,
                          scores ? scores + int64_t(r0) * ld_idx : nullptr, ld_idx, st);
        if (s != DSA_OK) return s;
    }
    return DSA_OK;
}

// ------------------------------------------------------ tensor-core path

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled from the driver, found through the runtime (no link against libcuda).
EncodeTiledFn encode_tiled()
{
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Tensor map of a row-major [rows, D] bf16 matrix, loaded in boxes of box_rows
// rows x (64 or 128 bytes) with the matching shared-memory swizzle; rows past
// the end read as zeros.
bool make_tile_map(CUtensorMap* m, const void* base, int64_t rows, int D, int box_rows)
{
    EncodeTiledFn enc = encode_tiled();
    if (!enc || rows <= 0 || rows > INT32_MAX) return false;
    const int row_bytes = D * 2 >= 128 ? 128 : 64;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {(cuuint32_t)(row_bytes / 2), (cuuint32_t)box_rows};
    cuuint32_t elem[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, elem,
               CU_TENSOR_MAP_INTERLEAVE_NONE, row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int32_t tc_tile_rows(int H) { return 2 * (256 / H); }

int32_t tc_count_tiles(const int32_t* off, int n_seqs, int64_t row_base, int64_t n_rows, int32_t TQ)
{
    int64_t n = 0;
    for (int b = 0; b < n_seqs; ++b) {
        const int64_t lo = std::max<int64_t>(off[b], row_base), hi = std::min<int64_t>(off[b + 1], row_base + n_rows);
        if (hi > lo) n += (hi - lo + TQ - 1) / TQ;
    }
    return (int32_t)n;
}

// Key-range splits per query tile when there are fewer tiles than SMs (decode).  Units keep at
// least min_tiles key tiles (8 for the dense scan; HISA's short rows use 1 and 2).
int32_t tc_splits(int32_t tiles, int32_t max_cols, int32_t min_tiles = 8)
{
    const int32_t kt = (max_cols + 127) / 128;
    if (tiles <= 0 || tiles >= 148 || kt < 2 * min_tiles) return 1;
    // One CTA fills an SM, so the units run in waves of 148: pick the split count s (units of at
    // least min_tiles key tiles) minimising waves(s) * (ceil(kt / s) + 2), the 2 standing for a
    // CTA's start-up (barriers, TMEM, the query tile) in key tiles.
    int32_t best = 1;
    int64_t best_cost = INT64_MAX;
    for (int32_t s = 1; s <= kt / min_tiles; ++s) {
        const int64_t waves = (int64_t(tiles) * s + 147) / 148;
        const int64_t cost = waves * ((kt + s - 1) / s + 2);
        if (cost < best_cost) { best_cost = cost; best = s; }
    }
    return best;
}

// A query-row source for the tensor-core path: rows r of the launch read
// Q[rd.qrow] / W[rd.qrow]; seq_off are absolute row offsets of the segments
// (runs of rows that share one column -> key map: sequences, PIVOT groups or
// single HISA queries), with a host copy for sizing.
struct TcSource {
    const void* Q;
    int64_t q_rows;
    const float* W;
    const int32_t* seq_off;
    const int32_t* seq_off_host;
    int32_t n_seqs;
};

int32_t tc_unit_capacity(const TcSource& src, int32_t n_rows, int32_t chunk, int H, int32_t max_cols)
{
    const int32_t TQ = tc_tile_rows(H);
    int32_t cap = 1;
    for (int32_t r0 = 0; r0 < n_rows; r0 += chunk) {
        const int32_t nr = std::min(chunk, n_rows - r0);
        const int32_t t = tc_count_tiles(src.seq_off_host, src.n_seqs, r0, nr, TQ);
        cap = std::max(cap, t * tc_splits(t, max_cols));
    }
    return cap;
}

template <int D, int H>
dsa_status launch_tc_shape(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mkg, const TcArgs& a,
                           const DenseSetupArgs& su, int32_t n_units, int n_acc, cudaStream_t st)
{
    using SH = TcShape<D, H>;
    const int budget = 232448;
    int stages = (budget - (int)SH::smem_bytes(n_acc, 0)) / (int)SH::KTILE;
    stages = std::min(stages, kTcMaxStages);
    if (stages < 2) return DSA_ERR_UNSUPPORTED;
    TcArgs args = a;
    args.n_stages = stages;
    // >= 120 KB keeps one CTA per SM, so no two CTAs ever wait on each other for the 512 TMEM columns.
    const int smem = std::max((int)SH::smem_bytes(n_acc, stages), 120 * 1024);
    dsa_status s;
    if (a.gather) {
        if ((s = set_smem(score_tc_kernel<D, H, kTcGather>, smem)) != DSA_OK) return s;
        DSA_LAUNCH(kProfScoreTc, st, launch_pdl(latency_bound(n_units), score_tc_kernel<D, H, kTcGather>, n_units,
                                                kTcThreads, smem, st, mq, mk, mkg, args, su));
    } else if (a.planes > 1 || a.block_tiles) {
        if ((s = set_smem(score_tc_kernel<D, H, kTcBlocks>, smem)) != DSA_OK) return s;
        DSA_LAUNCH(kProfScoreTc, st, launch_pdl(latency_bound(n_units), score_tc_kernel<D, H, kTcBlocks>, n_units,
                                                kTcThreadsTiles, smem, st, mq, mk, mkg, args, su));
    } else {
        if ((s = set_smem(score_tc_kernel<D, H, kTcTiles>, smem)) != DSA_OK) return s;
        DSA_LAUNCH(kProfScoreTc, st, launch_pdl(latency_bound(n_units), score_tc_kernel<D, H, kTcTiles>, n_units,
                                                kTcThreadsTiles, smem, st, mq, mk, mkg, args, su));
    }
    return launched();
}

template <int D>
dsa_status launch_tc_d(int H, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mkg, const TcArgs& a,
                       const DenseSetupArgs& su, int32_t n_units, int n_acc, cudaStream_t st)
{
    switch (H) {
    case 1: return launch_tc_shape<D, 1>(mq, mk, mkg, a, su, n_units, n_acc, st);
    case 2: return launch_tc_shape<D, 2>(mq, mk, mkg, a, su, n_units, n_acc, st);
    case 4: return launch_tc_shape<D, 4>(mq, mk, mkg, a, su, n_units, n_acc, st);
    case 8: return launch_tc_shape<D, 8>(mq, mk, mkg, a, su, n_units, n_acc, st);
    case 16: return launch_tc_shape<D, 16>(mq, mk, mkg, a, su, n_units, n_acc, st);
    case 32: return launch_tc_shape<D, 32>(mq, mk, mkg, a, su, n_units, n_acc, st);
    default: return launch_tc_shape<D, 64>(mq, mk, mkg, a, su, n_units, n_acc, st);
    }
}

// Options of a tensor-core scoring launch.
struct TcOpts {
    bool units_ready = false;   // a set-up kernel already wrote the work units
    int32_t planes = 1;         // 3: K holds three bf16 planes of fp32 keys, plane_rows rows apart
    int64_t plane_rows = 0;
    int32_t min_tiles = 8;      // key tiles per unit at least (tc_splits)
    const DenseSetupArgs* own_setup = nullptr;   // dense launches of one wave: the kernel's own set-up
};

// Key tiles of a block map with whole 128-key tiles per block are contiguous: one tile load each.
bool block_tiles(const ColMap& m) { return m.kind == kMapBlocks && m.block % 128 == 0; }

// Tensor-core scores of launch rows [0, n_rows) (absolute [row_base, ...)) into
// S[r * ld + c] for the eligible columns c < rows[r].ncols; column c is key
// map(c) of the row's sequence.
dsa_status tc_score(const RowDesc* rows, int32_t n_rows, int32_t row_base, const TcSource& src, int H, int D,
                    const void* K, int64_t n_k, const int32_t* k_base, const ColMap& map, int32_t max_cols, float* S,
                    int64_t ld, TcUnit* units, int32_t* tile_base, uint32_t* status, cudaStream_t st,
                    const TcOpts& o = TcOpts{})
{
    if (n_rows <= 0 || max_cols <= 0 || n_k <= 0) return DSA_OK;
    const int32_t TQ = tc_tile_rows(H);
    const int32_t tiles = tc_count_tiles(src.seq_off_host, src.n_seqs, row_base, n_rows, TQ);
    if (tiles == 0) return DSA_OK;
    const int32_t splits = tc_splits(tiles, max_cols, o.min_tiles);
    const bool btiles = block_tiles(map);
    const bool gather = (map.kind != kMapIdentity || map.offset != 0) && !btiles;
    const bool units_ready = o.units_ready;
    CUtensorMap mq, mk, mkg;
    if (!make_tile_map(&mq, src.Q, src.q_rows * H, D, 256) || !make_tile_map(&mk, K, n_k, D, 128) ||
        !make_tile_map(&mkg, K, n_k, D, 1))
        return DSA_ERR_CUDA;
    if (!units_ready) {   // (else dense_setup_kernel wrote them)
        DSA_LAUNCH(kProfSetup, st, launch_pdl(latency_bound(int64_t(tiles) * splits), tc_units_kernel, 1, 1024, 0, st,
                                              rows, n_rows, row_base, src.seq_off, src.n_seqs, TQ, splits, k_base,
                                              tile_base, units));
        dsa_status s = launched();
        if (s != DSA_OK) return s;
    }
    int32_t max_q = 0;
    for (int b = 0; b < src.n_seqs; ++b) max_q = std::max(max_q, src.seq_off_host[b + 1] - src.seq_off_host[b]);
    const int n_acc = std::min(max_q, TQ) > TQ / 2 ? 2 : 1;
    TcArgs a{};
    a.units = units;
    a.rows = rows;
    a.map = map;
    a.gather = gather ? 1 : 0;
    // keys are read by several units: gathered candidate lists (shared by a segment's tiles and
    // by neighbouring segments) and the causal prefixes of prefill (one per query tile)
    a.keep_keys = gather || tiles > src.n_seqs ? 1 : 0;
    a.W = src.W;
    a.S = S;
    a.ld_s = ld;
    a.status = status;
    a.n_keys = n_k;
    a.planes = o.planes;
    a.plane_rows = o.plane_rows;
    a.block_tiles = btiles ? 1 : 0;
    static const DenseSetupArgs kNoSetup{};
    const DenseSetupArgs& su = o.own_setup ? *o.own_setup : kNoSetup;
    switch (D) {
    case 32: return launch_tc_d<32>(H, mq, mk, mkg, a, su, tiles * splits, n_acc, st);
    case 64: return launch_tc_d<64>(H, mq, mk, mkg, a, su, tiles * splits, n_acc, st);
    default: return launch_tc_d<128>(H, mq, mk, mkg, a, su, tiles * splits, n_acc, st);
    }
}

// Tensor-core scoring then exact top-k, in row chunks that fit the score buffer.
dsa_status tc_score_and_select(const RowDesc* rows, int32_t n_rows, const TcSource& src, int H, int D, const void* K,
                               int64_t n_k, const int32_t* k_base, const ColMap& map, int32_t max_cols, float* Sbuf,
                               TcUnit* units, int32_t* tile_base, uint32_t* status, int32_t k, int32_t* idx,
                               int64_t ld_idx, float* scores, cudaStream_t st, const SelectSplit& sp = SelectSplit{})
{
    const int64_t ld = score_ld(max_cols);
    const int32_t chunk = chunk_rows(n_rows, ld);
    for (int32_t r0 = 0; r0 < n_rows; r0 += chunk) {
        const int32_t nr = std::min(chunk, n_rows - r0);
        dsa_status s = tc_score(rows + r0, nr, r0, src, H, D, K, n_k, k_base, map, max_cols, Sbuf, ld, units,
                                tile_base, status, st);
        if (s != DSA_OK) return s;
        s = launch_select(rows + r0, nr, max_cols, k, map, Sbuf, ld, false, idx + int64_t(r0) * ld_idx, ld_idx,
                          scores ? scores + int64_t(r0) * ld_idx : nullptr, ld_idx, st, sp);
        if (s != DSA_OK) return s;
    }
    return DSA_OK;
}

ColMap identity_map(int32_t offset = 0)
{
    ColMap m{};
    m.kind = kMapIdentity;
    m.offset = offset;
    return m;
}

// ------------------------------------------------------- workspace plans

struct DensePlan {
    RowDesc* rows;
    float* S;
    TcUnit* units;
    int32_t* tile_base;
    SelectSplit split;
};

// k = 0: the scores-only entry point (no score buffer, no select).  max_chunk: the caller scores
// at most this many rows at a time (the score buffer is sized for it).
size_t dense_plan(char* base, const dsa_batch* b, const HostInfo& hi, int32_t k, DensePlan* p,
                  int32_t max_chunk = INT32_MAX)
{
    Carver c{base};
    const int32_t nq = std::max(1, b->num_queries);
    p->rows = c.take<RowDesc>(nq);
    const int64_t ld = score_ld(hi.max_k);
    const int32_t chunk = k == 0 ? nq : std::min(max_chunk, chunk_rows(nq, ld));
    const TcSource src{nullptr, 0, nullptr, nullptr, b->q_offsets_host, b->num_seqs};
    p->units = c.take<TcUnit>(tc_unit_capacity(src, b->num_queries, chunk, b->num_heads, hi.max_k));
    p->tile_base = c.take<int32_t>(b->num_seqs + 1);
    p->split = SelectSplit{};
    if (k > 0) {
        p->S = c.take<float>(size_t(chunk) * ld);
        p->split.max_rows = split_rows_for(chunk);
        p->split.buf = c.take<uint64_t>(size_t(p->split.max_rows) * select_cap(k, hi.max_k));
        if (base) p->split.ctr = split_counters(base);
    }
    return c.off;
}

// Workspace of dsa_index_topk_host: dsa_index_topk's workspace first (its header stays at the
// base), then device copies of the inputs and kHostBufs row chunks' queries and indices.
constexpr int kHostBufs = 3;
constexpr int32_t kHostChunks = 8;        // row chunks a large batch is cut into
constexpr int32_t kHostMinChunk = 2048;   // rows per chunk at least

struct HostPlan {
    int32_t* q_off;
    int32_t* k_off;
    int32_t* q_pos;
    uint8_t* K;
    float* W;
    uint8_t* Q[kHostBufs];
    int32_t* idx[kHostBufs];
    RowDesc* rows;   // one chunk's rows, query rows relative to the chunk
    int32_t chunk;
};

// Rows per chunk of the host-memory entry point: about kHostChunks chunks of at least kHostMinChunk
// rows (the copies of one chunk then overlap the work of another), and no more than the score
// buffer holds.
int32_t host_chunk_rows(int32_t nq, int64_t ld)
{
    const int32_t want = std::max(kHostMinChunk, (nq + kHostChunks - 1) / kHostChunks);
    return std::max(1, std::min(chunk_rows(nq, ld), want));
}

size_t host_plan(char* base, const dsa_batch* b, const HostInfo& hi, int32_t k, DensePlan* dp, HostPlan* p)
{
    const size_t inner = dense_plan(base, b, hi, k, dp,
                                    host_chunk_rows(std::max(1, b->num_queries), score_ld(hi.max_k)));
    Carver c{base};
    c.off = align256(inner);
    const int32_t nq = std::max(1, b->num_queries);
    const size_t qrow_bytes = size_t(b->num_heads) * b->head_dim * 2;
    p->chunk = host_chunk_rows(nq, score_ld(hi.max_k));
    p->q_off = c.take<int32_t>(b->num_seqs + 1);
    p->k_off = c.take<int32_t>(b->num_seqs + 1);
    p->q_pos = c.take<int32_t>(nq);
    p->K = c.take<uint8_t>(size_t(std::max(1, b->num_keys)) * b->head_dim * 2);
    p->W = c.take<float>(size_t(nq) * b->num_heads);
    for (int i = 0; i < kHostBufs; ++i) {
        p->Q[i] = c.take<uint8_t>(size_t(p->chunk) * qrow_bytes);
        p->idx[i] = c.take<int32_t>(size_t(p->chunk) * k);
    }
    p->rows = c.take<RowDesc>(p->chunk);
    return c.off;
}

struct PivotPlan {
    int32_t* group_base;
    GroupDesc* groups;
    RowDesc* proxy_rows;
    RowDesc* query_rows;
    __nv_bfloat16* Qp;
    float* Wp;
    int32_t* cand;
    float* cand_score;
    float* S;
    TcUnit* units;
    int32_t* tile_base;
    int32_t* group_rows;   // [n_groups + 1] first query row of each group
    // Reuse: the group's top k + G - 1 candidates, and the queries that need their own selection
    RowDesc* cand_rows;    // [n_groups]
    int32_t* gsel;         // [n_groups, kp]
    float* gscore;         // [n_groups, kp]
    RowDesc* fb_rows;      // [n_q]
};

// Reuse's group list length: k plus the most candidates a query of a group with consecutive
// positions can lose to its own causal limit.
int32_t reuse_list_len(int32_t k, int32_t G, int32_t C) { return std::min(k + G - 1, C); }

int32_t count_groups(const dsa_batch* b, int32_t G)
{
    int64_t n = 0;
    for (int i = 0; i < b->num_seqs; ++i)
        n += (b->q_offsets_host[i + 1] - b->q_offsets_host[i] + G - 1) / G;
    return (int32_t)n;
}

// Host copy of the per-sequence group offsets (what pivot_groups_kernel writes on the device).
std::vector<int32_t> group_offsets_host(const dsa_batch* b, int32_t G)
{
    std::vector<int32_t> off(b->num_seqs + 1, 0);
    for (int i = 0; i < b->num_seqs; ++i)
        off[i + 1] = off[i] + (b->q_offsets_host[i + 1] - b->q_offsets_host[i] + G - 1) / G;
    return off;
}

// Host copy of the query-row offsets of every group (what group_row_offsets_kernel writes).
std::vector<int32_t> group_rows_host(const dsa_batch* b, int32_t G)
{
    std::vector<int32_t> off;
    for (int i = 0; i < b->num_seqs; ++i)
        for (int32_t r = b->q_offsets_host[i]; r < b->q_offsets_host[i + 1]; r += G) off.push_back(r);
    off.push_back(b->num_queries);
    return off;
}

size_t pivot_plan(char* base, const dsa_batch* b, const HostInfo& hi, int32_t k, int32_t G, int32_t C, int32_t mode,
                  PivotPlan* p)
{
    Carver c{base};
    const int32_t ng = std::max(1, count_groups(b, G));
    p->group_base = c.take<int32_t>(b->num_seqs + 1);
    p->groups = c.take<GroupDesc>(ng);
    p->proxy_rows = c.take<RowDesc>(ng);
    p->query_rows = c.take<RowDesc>(std::max(1, b->num_queries));
    p->Qp = c.take<__nv_bfloat16>(size_t(ng) * b->num_heads * b->head_dim);
    p->Wp = c.take<float>(size_t(ng) * b->num_heads);
    p->cand = c.take<int32_t>(size_t(ng) * C);
    p->cand_score = c.take<float>(size_t(ng) * C);
    const int64_t ld_scan = score_ld(hi.max_k), ld_ref = score_ld(C);
    const int32_t chunk_scan = chunk_rows(ng, ld_scan);
    const size_t s_scan = size_t(chunk_scan) * ld_scan;
    const size_t s_ref = size_t(chunk_rows(std::max(1, b->num_queries), ld_ref)) * ld_ref;
    p->S = c.take<float>(mode == 0 ? s_scan : std::max(s_scan, s_ref));
    const std::vector<int32_t> goff = group_offsets_host(b, G);
    const TcSource src{nullptr, 0, nullptr, nullptr, goff.data(), b->num_seqs};
    const std::vector<int32_t> groff = group_rows_host(b, G);
    const TcSource srf{nullptr, 0, nullptr, nullptr, groff.data(), (int32_t)groff.size() - 1};
    const int32_t cap = std::max(tc_unit_capacity(src, count_groups(b, G), chunk_scan, b->num_heads, hi.max_k),
                                 tc_unit_capacity(srf, b->num_queries, chunk_rows(std::max(1, b->num_queries), ld_ref),
                                                  b->num_heads, C));
    p->units = c.take<TcUnit>(cap);
    p->tile_base = c.take<int32_t>(std::max(b->num_seqs, ng) + 1);
    p->group_rows = c.take<int32_t>(ng + 1);
    p->cand_rows = nullptr;
    p->gsel = nullptr;
    p->gscore = nullptr;
    p->fb_rows = nullptr;
    if (mode == 0) {
        const int32_t kp = reuse_list_len(k, G, C);
        p->cand_rows = c.take<RowDesc>(ng);
        p->gsel = c.take<int32_t>(size_t(ng) * kp);
        p->gscore = c.take<float>(size_t(ng) * kp);
        p->fb_rows = c.take<RowDesc>(std::max(1, b->num_queries));
    }
    return c.off;
}

// Count of the Reuse queries left to the per-query selection: a word of the workspace's
// status area, which every call clears before its first launch.
int32_t* reuse_fallback_count(void* ws) { return reinterpret_cast<int32_t*>(static_cast<char*>(ws) + 64); }

// Reuse without a candidate list: the groups the gated top-C selection ranks (0, or all of them once
// some query needs the per-query selection); the next word of the status area.
int32_t* reuse_gate(void* ws) { return reinterpret_cast<int32_t*>(static_cast<char*>(ws) + 68); }

struct HisaPlan {
    int32_t* block_base;
    RowDesc* block_rows;
    RowDesc* token_rows;
    int32_t* mid;
    int32_t* kept;
    float* S;
    int32_t* query_off;    // [n_q + 1] 0..n_q: every query is its own segment
    TcUnit* units;
    int32_t* tile_base;
    SelectSplit split;     // the token stage's select
    uint32_t* planes;      // the pooled keys as three bf16 planes (one-pass step)
    TcUnit* block_units;   // the block stage's scoring units (one-pass step)
};

std::vector<int32_t> iota_host(int32_t n)
{
    std::vector<int32_t> v(n + 1);
    for (int32_t i = 0; i <= n; ++i) v[i] = i;
    return v;
}

// Sizes of HISA's one-pass step (hisa_one_pass): pooled blocks, the block stage's query tiles
// and key-range splits (units of one key tile of 128 blocks), and the token stage's splits
// (units of at least two key tiles; every query is its own segment).
struct HisaShape {
    int64_t blocks;
    int32_t max_mid;
    int32_t tok_cols;
    int32_t block_tiles;
    int32_t block_splits;
    int32_t token_splits;
};

HisaShape hisa_shape(const dsa_batch* b, const HostInfo& hi, int32_t B, int32_t keep)
{
    HisaShape h{};
    for (int i = 0; i < b->num_seqs; ++i) h.blocks += (b->k_offsets_host[i + 1] - b->k_offsets_host[i] + B - 1) / B;
    h.max_mid = std::max(0, (hi.max_k + B - 1) / B - 2);
    h.tok_cols = (keep + 2) * B;
    h.block_tiles = tc_count_tiles(b->q_offsets_host, b->num_seqs, 0, b->num_queries, tc_tile_rows(b->num_heads));
    h.block_splits = tc_splits(h.block_tiles, h.max_mid, 1);
    h.token_splits = tc_splits(b->num_queries, h.tok_cols, 2);
    return h;
}

// Rows the register top-k takes (one CTA of up to 1024 threads, 16 columns each).
constexpr int32_t kRegsMaxCols = 16384;

// Whether a HISA call runs as the one-pass step: the sequences' tile offsets fit the set-up's
// argument block, both stages' rows fit the register top-k, and both stages' scores fit the score
// buffer at once.
bool hisa_one_pass_ok(const dsa_batch* b, const HostInfo& hi, int32_t B, int32_t keep)
{
    const int32_t nq = b->num_queries;
    if (nq <= 0 || b->num_seqs > kSetupMaxSeqs) return false;
    const HisaShape h = hisa_shape(b, hi, B, keep);
    if (h.max_mid > kRegsMaxCols || h.tok_cols > kRegsMaxCols || 3 * h.blocks > INT32_MAX) return false;
    return chunk_rows(nq, score_ld(h.max_mid)) >= nq && chunk_rows(nq, score_ld(h.tok_cols)) >= nq;
}

size_t hisa_plan(char* base, const dsa_batch* b, const HostInfo& hi, int32_t k, int32_t B, int32_t keep, HisaPlan* p)
{
    Carver c{base};
    const int32_t nq = std::max(1, b->num_queries);
    p->block_base = c.take<int32_t>(b->num_seqs + 1);
    p->block_rows = c.take<RowDesc>(nq);
    p->token_rows = c.take<RowDesc>(nq);
    p->mid = c.take<int32_t>(size_t(nq) * keep);
    p->kept = c.take<int32_t>(size_t(nq) * (keep + 2));
    const int32_t max_mid = std::max(0, (hi.max_k + B - 1) / B - 2);   // as hisa_index scores them
    const int64_t ld_blk = score_ld(max_mid), ld_tok = score_ld((keep + 2) * B);
    const size_t s_blk = size_t(chunk_rows(nq, ld_blk)) * ld_blk;
    const size_t s_tok = size_t(chunk_rows(nq, ld_tok)) * ld_tok;
    p->S = c.take<float>(std::max(s_blk, s_tok));
    p->query_off = c.take<int32_t>(nq + 1);
    const std::vector<int32_t> qoff = iota_host(b->num_queries);
    const TcSource src{nullptr, 0, nullptr, nullptr, qoff.data(), b->num_queries};
    p->units = c.take<TcUnit>(tc_unit_capacity(src, b->num_queries, chunk_rows(nq, ld_tok), b->num_heads,
                                                  (keep + 2) * B));
    p->tile_base = c.take<int32_t>(nq + 1);
    p->split = SelectSplit{};
    p->split.max_rows = split_rows_for(chunk_rows(nq, ld_tok));
    p->split.buf = c.take<uint64_t>(size_t(p->split.max_rows) * select_cap(k, (keep + 2) * B));
    if (base) p->split.ctr = split_counters(base);
    if (hisa_one_pass_ok(b, hi, B, keep)) {
        const HisaShape h = hisa_shape(b, hi, B, keep);
        p->planes = c.take<uint32_t>(size_t(3) * h.blocks * b->head_dim / 2);
        p->block_units = c.take<TcUnit>(size_t(h.block_tiles) * h.block_splits);
        p->units = c.take<TcUnit>(size_t(nq) * h.token_splits);   // (replaces the chunked path's table)
    } else {
        p->planes = nullptr;
        p->block_units = nullptr;
    }
    return c.off;
}

dsa_status clear_status(void* ws, cudaStream_t st)
{
    g_status = static_cast<uint32_t*>(ws);
    return cudaMemsetAsync(ws, 0, kHeaderBytes, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// dsa_index_topk for a batch scored in one launch (decode; prefill within the score buffer): one
// set-up kernel (the header cleared, rows, work units), the scoring launch, the select: three
// launches, the later two programmatic where their grids are small.
dsa_status dense_topk_one_launch(const dsa_batch* b, const HostInfo& hi, const TcSource& src, const void* K,
                                 int32_t k, int32_t* idx, float* scores, const DensePlan& p, void* ws,
                                 cudaStream_t st)
{
    static_assert(kHeaderBytes % 4 == 0, "header words");
    const int32_t TQ = tc_tile_rows(b->num_heads);
    g_status = static_cast<uint32_t*>(ws);
    DenseSetupArgs a{};
    a.q_off = b->q_offsets;
    a.k_off = b->k_offsets;
    a.q_pos = b->q_pos;
    a.rows = p.rows;
    a.units = p.units;
    a.header = static_cast<uint32_t*>(ws);
    a.header_words = (int32_t)(kHeaderBytes / 4);
    a.n_seqs = b->num_seqs;
    a.n_q = b->num_queries;
    a.TQ = TQ;
    int32_t tiles = 0;
    for (int i = 0; i < b->num_seqs; ++i) {
        a.tile_base[i] = tiles;
        tiles += (b->q_offsets_host[i + 1] - b->q_offsets_host[i] + TQ - 1) / TQ;
    }
    a.tile_base[b->num_seqs] = tiles;
    a.splits = tc_splits(tiles, hi.max_k);   // as tc_score derives it
    a.n_units = tiles * a.splits;
    TcOpts o;
    o.units_ready = true;
    dsa_status s;
    if (a.n_units <= 148) {
        // one wave (decode): the scoring kernel sets itself up (every query row is in some unit's tile)
        o.own_setup = &a;
    } else {
        const int grid = (std::max(a.n_q, a.n_units) + 255) / 256;
        // a plain launch: it starts once the stream's earlier work (which may use this workspace) is done
        DSA_LAUNCH(kProfSetup, st, launch_pdl(false, dense_setup_kernel, grid, 256, 0, st, a));
        if ((s = launched()) != DSA_OK) return s;
    }
    const int64_t ld = score_ld(hi.max_k);
    uint32_t* status = static_cast<uint32_t*>(ws);
    s = tc_score(p.rows, b->num_queries, 0, src, b->num_heads, b->head_dim, K, b->num_keys, b->k_offsets, ColMap{},
                 hi.max_k, p.S, ld, p.units, p.tile_base, status, st, o);
    if (s != DSA_OK) return s;
    return launch_select(p.rows, b->num_queries, hi.max_k, k, ColMap{}, p.S, ld, false, idx, k, scores, k, st, p.split);
}

// PIVOT Reuse when the caller wants no candidate list (pivot_group_index, mode 0, cand NULL).  The
// scan's scores stay in the buffer; the group's top k + G - 1 are selected from the proxy row
// directly (no top-C selection); the Reuse kernel serves every query whose prefix keeps k of them.
// Only if some query is left over (ragged positions) does a gated top-C selection build the
// candidate lists, after which those queries are ranked one by one as in the listed path.
dsa_status reuse_direct(const dsa_batch* b, const HostInfo& hi, const void* K, int32_t k, int32_t G, int32_t C,
                        int32_t ng, const TcSource& src, int32_t* idx, const PivotPlan& p, void* ws, cudaStream_t st)
{
    uint32_t* status = static_cast<uint32_t*>(ws);
    const int64_t ld = score_ld(hi.max_k);
    dsa_status s = tc_score(p.proxy_rows, ng, 0, src, b->num_heads, b->head_dim, K, b->num_keys, b->k_offsets,
                            ColMap{}, hi.max_k, p.S, ld, p.units, p.tile_base, status, st);
    if (s != DSA_OK) return s;
    const int32_t kp = reuse_list_len(k, G, C);
    if ((s = launch_select(p.proxy_rows, ng, hi.max_k, kp, identity_map(), p.S, ld, false, p.gsel, kp, p.gscore, kp,
                           st)) != DSA_OK)
        return s;
    const unsigned gq = (b->num_queries + 255) / 256;
    DSA_LAUNCH(kProfSetup, st, pivot_query_rows_kernel<<<gq, 256, 0, st>>>(b->q_offsets, b->k_offsets, b->q_pos,
                                                                           b->num_seqs, b->num_queries, G, p.group_base,
                                                                           nullptr, C, nullptr, p.query_rows));
    if ((s = launched()) != DSA_OK) return s;
    DSA_LAUNCH(kProfSetup, st, pivot_cand_rows_kernel<<<(ng + 255) / 256, 256, 0, st>>>(p.groups, ng, C, p.cand_rows));
    if ((s = launched()) != DSA_OK) return s;
    ReuseArgs ra{};
    ra.groups = p.groups; ra.query_rows = p.query_rows; ra.cand_rows = p.cand_rows;
    ra.gsel = p.gsel; ra.gscore = p.gscore; ra.kp = kp; ra.k = k; ra.cand = nullptr; ra.C = C;
    ra.n_groups = ng; ra.gate = reuse_gate(ws);
    ra.idx = idx; ra.ld_idx = k; ra.fb_rows = p.fb_rows; ra.fb_count = reuse_fallback_count(ws);
    ra.status = status;
    const size_t smem = reuse_smem_bytes(kp);
    if ((s = set_smem(pivot_reuse_kernel, smem)) != DSA_OK) return s;
    DSA_LAUNCH(kProfSelect, st, pivot_reuse_kernel<<<ng, kReuseThreads, smem, st>>>(ra));
    if ((s = launched()) != DSA_OK) return s;
    // left-over queries: the candidate lists (every group, or none when the gate stayed shut), their rows, their top k
    if ((s = launch_select(p.proxy_rows, ng, hi.max_k, C, identity_map(), p.S, ld, false, p.cand, C, p.cand_score, C,
                           st, SelectSplit{}, reuse_gate(ws))) != DSA_OK)
        return s;
    DSA_LAUNCH(kProfSetup, st, reuse_fallback_rows_kernel<<<gq, 256, 0, st>>>(p.fb_rows, reuse_fallback_count(ws),
                                                                              p.cand, C));
    if ((s = launched()) != DSA_OK) return s;
    ColMap m{};
    m.kind = kMapList;
    m.list = p.cand;
    m.list_ld = C;
    return launch_select(p.fb_rows, b->num_queries, C, k, m, p.cand_score, C, true, idx, k, nullptr, 0, st,
                         SelectSplit{}, reuse_fallback_count(ws));
}

// PIVOT Refine's second stage: each query scores its eligible candidates (query_rows, list map m)
// with its own indexer on tensor cores, the group's candidate keys gathered tile by tile.
dsa_status refine_stage(const dsa_batch* b, const void* Q, const void* K, const float* W, int32_t k, int32_t G,
                        int32_t C, int32_t ng, const ColMap& m, int32_t* idx, const PivotPlan& p, void* ws,
                        cudaStream_t st)
{
    DSA_LAUNCH(kProfSetup, st, group_row_offsets_kernel<<<(ng + 256) / 256, 256, 0, st>>>(p.groups, ng, b->num_queries,
                                                                                          p.group_rows));
    dsa_status s;
    if ((s = launched()) != DSA_OK) return s;
    const std::vector<int32_t> groff = group_rows_host(b, G);
    const TcSource srf{Q, b->num_queries, W, p.group_rows, groff.data(), ng};
    return tc_score_and_select(p.query_rows, b->num_queries, srf, b->num_heads, b->head_dim, K, b->num_keys,
                               b->k_offsets, m, C, p.S, p.units, p.tile_base, static_cast<uint32_t*>(ws), k, idx, k,
                               nullptr, st);
}

template <int NT, int R>
struct RegsHisaBlocks {
    static dsa_status run(size_t smem, int32_t n_rows, const SelectArgs& a, const HisaKeptArgs& h, cudaStream_t st)
    {
        dsa_status s = set_smem(hisa_block_select_kernel<NT, R>, smem);
        if (s != DSA_OK) return s;
        DSA_LAUNCH(kProfSelect, st, launch_pdl(latency_bound(n_rows), hisa_block_select_kernel<NT, R>, n_rows, NT, smem,
                                               st, a, h));
        return launched();
    }
};

// HISA in one launch per stage (hisa_one_pass_ok): set-up (rows, block units, the pooled keys'
// bf16 planes), block scores on the tensor cores, block top-`keep` fused with the kept blocks, the
// token rows and the token units, token scores on the tensor cores (one tile load per kept block
// when blocks are whole key tiles), token top-k: five launches, the later four programmatic.
dsa_status hisa_one_pass(const dsa_batch* b, const HostInfo& hi, const void* Q, const void* K, const float* W,
                         const float* pooled, int32_t k, int32_t B, int32_t keep, int32_t* idx, int32_t* kept,
                         const HisaPlan& p, void* ws, cudaStream_t st)
{
    const int32_t nq = b->num_queries, H = b->num_heads, D = b->head_dim;
    const HisaShape h = hisa_shape(b, hi, B, keep);
    uint32_t* status = static_cast<uint32_t*>(ws);
    g_status = status;
    HisaSetupArgs a{};
    a.q_off = b->q_offsets;
    a.k_off = b->k_offsets;
    a.q_pos = b->q_pos;
    a.pooled = pooled;
    a.planes = p.planes;
    a.rows = p.block_rows;
    a.units = p.block_units;
    a.query_off = p.query_off;
    a.header = status;
    a.header_words = (int32_t)(kHeaderBytes / 4);
    a.n_seqs = b->num_seqs;
    a.n_q = nq;
    a.B = B;
    a.TQ = tc_tile_rows(H);
    int32_t tiles = 0, blocks = 0;
    for (int i = 0; i < b->num_seqs; ++i) {
        a.tile_base[i] = tiles;
        a.block_base[i] = blocks;
        tiles += (b->q_offsets_host[i + 1] - b->q_offsets_host[i] + a.TQ - 1) / a.TQ;
        blocks += (b->k_offsets_host[i + 1] - b->k_offsets_host[i] + B - 1) / B;
    }
    a.tile_base[b->num_seqs] = tiles;
    a.block_base[b->num_seqs] = blocks;
    a.splits = h.block_splits;
    a.n_units = h.block_tiles * h.block_splits;
    a.n_pairs = int64_t(blocks) * D / 2;
    a.row_ctas = (std::max(nq + 1, a.n_units) + 255) / 256;
    const int split_ctas = (int)std::min<int64_t>(2 * 148, (a.n_pairs + 255) / 256);
    DSA_LAUNCH(kProfSetup, st, launch_pdl(false, hisa_setup_tc_kernel, a.row_ctas + split_ctas, 256, 0, st, a));
    dsa_status s = launched();
    if (s != DSA_OK) return s;

    // Coarse stage: the middle blocks' pooled keys as three bf16 planes on the tensor cores.
    const TcSource bsrc{Q, nq, W, b->q_offsets, b->q_offsets_host, b->num_seqs};
    const int64_t ld_blk = score_ld(h.max_mid), ld_tok = score_ld(h.tok_cols);
    TcOpts ob;
    ob.units_ready = true;
    ob.planes = 3;
    ob.plane_rows = blocks;
    ob.min_tiles = 1;
    s = tc_score(p.block_rows, nq, 0, bsrc, H, D, p.planes, 3 * int64_t(blocks), nullptr, ColMap{}, h.max_mid, p.S,
                 ld_blk, p.block_units, p.tile_base, status, st, ob);
    if (s != DSA_OK) return s;
    SelectArgs sa{};
    sa.rows = p.block_rows;
    sa.n_rows = nq;
    sa.k = keep;
    sa.map = identity_map(1);   // column c is middle block c + 1
    sa.S = p.S;
    sa.ld_s = ld_blk;
    sa.status = status;
    const HisaKeptArgs ka{b->q_pos, b->k_offsets, B, keep, h.token_splits, 0, kept, p.token_rows, p.units};
    if ((s = launch_regs<RegsHisaBlocks>(h.max_mid, size_t(keep) * 4, nq, sa, ka, st)) != DSA_OK) return s;

    // Fine stage: the indexer over the tokens of the kept blocks, then the top k.
    ColMap m{};
    m.kind = kMapBlocks;
    m.block = B;
    m.list = kept;
    m.list_ld = keep + 2;
    const std::vector<int32_t> qoff = iota_host(nq);
    const TcSource tsrc{Q, nq, W, p.query_off, qoff.data(), nq};
    TcOpts ot;
    ot.units_ready = true;
    ot.min_tiles = 2;
    s = tc_score(p.token_rows, nq, 0, tsrc, H, D, K, b->num_keys, b->k_offsets, m, h.tok_cols, p.S, ld_tok, p.units,
                 p.tile_base, status, st, ot);
    if (s != DSA_OK) return s;
    SelectArgs ta{};
    ta.rows = p.token_rows;
    ta.n_rows = nq;
    ta.k = k;
    ta.map = m;
    ta.S = p.S;
    ta.ld_s = ld_tok;
    ta.status = status;
    ta.out_idx = idx;
    ta.ld_idx = k;
    return launch_regs<RegsSelect>(h.tok_cols, size_t(k) * 4, nq, ta, st);
}

}  // namespace

// =====================================================================
extern "C" {

const char* dsa_status_string(dsa_status s)
{
    switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape";
    case DSA_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_DEVICE_CHECK: return "a kernel recorded a device-side error";
    }
    return "unknown status";
}

int32_t dsa_version(void) { return 100; }

// ------------------------------------------------------------ dense scores
size_t dsa_index_scores_workspace(const dsa_batch* b)
{
    HostInfo hi;
    if (check_batch(b, &hi) != DSA_OK) return 0;
    DensePlan p;
    return dense_plan(nullptr, b, hi, 0, &p);
}

dsa_status dsa_index_scores(const dsa_batch* b, const void* Q, const void* K, const float* W, float* S,
                            int64_t ld_s, void* ws, size_t ws_bytes, void* stream)
{
    HostInfo hi;
    dsa_status s = check_batch(b, &hi);
    if (s != DSA_OK) return s;
    if ((s = check_tensors(b, Q, K, W)) != DSA_OK) return s;
    if (b->num_queries > 0 && (!S || ld_s < hi.max_k || ld_s > INT32_MAX)) return DSA_ERR_INVALID_ARG;
    DensePlan p;
    if ((s = check_ws(ws, ws_bytes, dense_plan(nullptr, b, hi, 0, &p))) != DSA_OK) return s;
    dense_plan(static_cast<char*>(ws), b, hi, 0, &p);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((s = clear_status(ws, st)) != DSA_OK) return s;
    if (b->num_queries == 0) return DSA_OK;
    DSA_LAUNCH(kProfSetup, st, dense_rows_kernel<<<(b->num_queries + 255) / 256, 256, 0, st>>>(b->q_offsets, b->k_offsets, b->q_pos,
                                                                    b->num_seqs, b->num_queries, p.rows));
    if ((s = launched()) != DSA_OK) return s;
    DSA_LAUNCH(kProfFill, st, fill_neg_inf_kernel<<<1184, 256, 0, st>>>(S, ld_s, b->num_queries, (int32_t)ld_s));
    if ((s = launched()) != DSA_OK) return s;
    const TcSource src{Q, b->num_queries, W, b->q_offsets, b->q_offsets_host, b->num_seqs};
    return tc_score(p.rows, b->num_queries, 0, src, b->num_heads, b->head_dim, K, b->num_keys, b->k_offsets, ColMap{},
                    hi.max_k,
                    S, ld_s, p.units, p.tile_base, static_cast<uint32_t*>(ws), st);
}

// ------------------------------------------------------------- dense top-k
size_t dsa_index_topk_workspace(const dsa_batch* b, int32_t k)
{
    HostInfo hi;
    if (check_batch(b, &hi) != DSA_OK || k < 1 || k > kMaxK) return 0;
    DensePlan p;
    return dense_plan(nullptr, b, hi, k, &p);
}

dsa_status dsa_index_topk(const dsa_batch* b, const void* Q, const void* K, const float* W, int32_t k,
                          int32_t* idx, float* scores, void* ws, size_t ws_bytes, void* stream)
{
    HostInfo hi;
    dsa_status s = check_batch(b, &hi);
    if (s != DSA_OK) return s;
    if (k < 1 || k > kMaxK || !select_fits(k, hi.max_k)) return DSA_ERR_UNSUPPORTED;
    if ((s = check_tensors(b, Q, K, W)) != DSA_OK) return s;
    if (b->num_queries > 0 && !idx) return DSA_ERR_INVALID_ARG;
    DensePlan p;
    if ((s = check_ws(ws, ws_bytes, dense_plan(nullptr, b, hi, k, &p))) != DSA_OK) return s;
    dense_plan(static_cast<char*>(ws), b, hi, k, &p);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const TcSource src{Q, b->num_queries, W, b->q_offsets, b->q_offsets_host, b->num_seqs};
    if (b->num_queries > 0 && b->num_keys > 0 && hi.max_k > 0 && b->num_seqs <= kSetupMaxSeqs &&
        chunk_rows(b->num_queries, score_ld(hi.max_k)) >= b->num_queries)
        return dense_topk_one_launch(b, hi, src, K, k, idx, scores, p, ws, st);
    if ((s = clear_status(ws, st)) != DSA_OK) return s;
    if (b->num_queries == 0) return DSA_OK;
    DSA_LAUNCH(kProfSetup, st, dense_rows_kernel<<<(b->num_queries + 255) / 256, 256, 0, st>>>(b->q_offsets, b->k_offsets, b->q_pos,
                                                                    b->num_seqs, b->num_queries, p.rows));
    if ((s = launched()) != DSA_OK) return s;
    return tc_score_and_select(p.rows, b->num_queries, src, b->num_heads, b->head_dim, K, b->num_keys, b->k_offsets,
                               ColMap{}, hi.max_k, p.S, p.units, p.tile_base, static_cast<uint32_t*>(ws), k, idx, k, scores, st,
                               p.split);
}

// ------------------------------------------------- cross-layer index reuse
int32_t dsa_index_layers_source(int32_t layer, int32_t retain_every, int32_t lag)
{
    if (layer < 0 || retain_every < 1 || (lag != 0 && lag != 1)) return -1;
    const int32_t consumer = lag == 1 && layer > 0 ? layer - 1 : layer;   // MLI: the previous layer's selection
    return consumer / retain_every * retain_every;                       // IndexCache: its nearest indexed layer
}

size_t dsa_index_layers_workspace(const dsa_batch* b, int32_t k) { return dsa_index_topk_workspace(b, k); }

dsa_status dsa_index_layers(const dsa_batch* b, int32_t n_layers, const void* const* Q, const void* const* K,
                            const float* const* W, int32_t k, int32_t retain_every, int32_t lag, int32_t* const* idx,
                            void* const* ready_events, void* ws, size_t ws_bytes, void* stream, void* side_stream)
{
    if (n_layers < 1 || retain_every < 1 || (lag != 0 && lag != 1) || !Q || !K || !W || !idx) return DSA_ERR_INVALID_ARG;
    if (!side_stream || side_stream == stream) return DSA_ERR_INVALID_ARG;
    HostInfo hi;
    dsa_status s = check_batch(b, &hi);
    if (s != DSA_OK) return s;
    for (int32_t l = 0; l < n_layers; ++l) {
        if (!idx[l]) return DSA_ERR_INVALID_ARG;
        if ((s = check_tensors(b, Q[l], K[l], W[l])) != DSA_OK) return s;
    }
    if (k < 1 || k > kMaxK || !select_fits(k, hi.max_k)) return DSA_ERR_UNSUPPORTED;
    if ((s = check_ws(ws, ws_bytes, dsa_index_topk_workspace(b, k))) != DSA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream), side = static_cast<cudaStream_t>(side_stream);
    cudaEvent_t ev_in, ev_out;
    if (cudaEventCreateWithFlags(&ev_in, cudaEventDisableTiming) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaEventCreateWithFlags(&ev_out, cudaEventDisableTiming) != cudaSuccess) {
        cudaEventDestroy(ev_in);
        return DSA_ERR_CUDA;
    }
    bool ok = true;
    auto chk = [&](cudaError_t e) { ok = ok && e == cudaSuccess; };
    // the side stream starts after the work already on `stream` (the layers' inputs)
    chk(cudaEventRecord(ev_in, st));
    chk(cudaStreamWaitEvent(side, ev_in, 0));
    const size_t row_bytes = size_t(std::max(b->num_queries, 0)) * k * sizeof(int32_t);
    // each indexed layer's top-k, written into its first consumer's rows and copied to the others
    for (int32_t f = 0; f < n_layers && ok && s == DSA_OK; f += retain_every) {
        int32_t first = -1;
        for (int32_t l = 0; l < n_layers; ++l) {
            if (dsa_index_layers_source(l, retain_every, lag) != f) continue;
            if (first < 0) {
                first = l;
                s = dsa_index_topk(b, Q[f], K[f], W[f], k, idx[l], nullptr, ws, ws_bytes, side);
                if (s != DSA_OK) break;
            } else if (row_bytes > 0) {
                chk(cudaMemcpyAsync(idx[l], idx[first], row_bytes, cudaMemcpyDeviceToDevice, side));
            }
            if (ready_events && ready_events[l]) chk(cudaEventRecord(static_cast<cudaEvent_t>(ready_events[l]), side));
        }
    }
    if (!ready_events) {   // without per-layer events, `stream` waits for every selection
        chk(cudaEventRecord(ev_out, side));
        chk(cudaStreamWaitEvent(st, ev_out, 0));
    }
    cudaEventDestroy(ev_in);
    cudaEventDestroy(ev_out);
    if (s != DSA_OK) return s;
    return ok ? DSA_OK : DSA_ERR_CUDA;
}

// ------------------------------------------------- dense top-k from host memory
size_t dsa_index_topk_host_workspace(const dsa_batch* b, int32_t k)
{
    dsa_batch d = *b;   // device pointers are the library's own copies here: any non-null stand-in
    d.q_offsets = d.k_offsets = d.q_pos = reinterpret_cast<const int32_t*>(b->q_offsets_host);
    HostInfo hi;
    if (check_batch(&d, &hi) != DSA_OK || k < 1 || k > kMaxK) return 0;
    DensePlan dp;
    HostPlan hp;
    return host_plan(nullptr, &d, hi, k, &dp, &hp);
}

dsa_status dsa_index_topk_host(const dsa_batch* b, const int32_t* q_pos_host, const void* Q, const void* K,
                               const float* W, int32_t k, int32_t* idx, void* ws, size_t ws_bytes, void* stream,
                               void* in_stream, void* out_stream)
{
    if (!b || !q_pos_host) return DSA_ERR_INVALID_ARG;
    dsa_batch d = *b;
    d.q_offsets = d.k_offsets = d.q_pos = reinterpret_cast<const int32_t*>(b->q_offsets_host);   // checked below
    HostInfo hi;
    dsa_status s = check_batch(&d, &hi);
    if (s != DSA_OK) return s;
    if (k < 1 || k > kMaxK || !select_fits(k, hi.max_k)) return DSA_ERR_UNSUPPORTED;
    if ((s = check_tensors(&d, Q, K, W)) != DSA_OK) return s;
    if (b->num_queries > 0 && !idx) return DSA_ERR_INVALID_ARG;
    if (stream == in_stream || stream == out_stream) return DSA_ERR_INVALID_ARG;
    DensePlan dp;
    HostPlan hp;
    if ((s = check_ws(ws, ws_bytes, host_plan(nullptr, &d, hi, k, &dp, &hp))) != DSA_OK) return s;
    host_plan(static_cast<char*>(ws), &d, hi, k, &dp, &hp);
    d.q_offsets = hp.q_off;
    d.k_offsets = hp.k_off;
    d.q_pos = hp.q_pos;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaStream_t si = static_cast<cudaStream_t>(in_stream), so = static_cast<cudaStream_t>(out_stream);
    if ((s = clear_status(ws, st)) != DSA_OK) return s;
    const int32_t nq = b->num_queries;
    if (nq == 0) return DSA_OK;
    const int H = b->num_heads, D = b->head_dim;
    const size_t qrow_bytes = size_t(H) * D * 2;

    // Row chunks in order of decreasing work (eligible pairs, from the host-side positions): the
    // largest are scored while the later chunks' queries still come in, and the last chunk, whose
    // work and index copy nothing overlaps, is the smallest (for a causal prefill, the first rows).
    const int32_t n_chunks = (nq + hp.chunk - 1) / hp.chunk;
    auto rows_of = [&](int32_t c) { return std::min(hp.chunk, nq - c * hp.chunk); };
    std::vector<int64_t> work(n_chunks, 0);
    for (int32_t q = 0; q < b->num_seqs; ++q) {
        const int32_t L = b->k_offsets_host[q + 1] - b->k_offsets_host[q];
        for (int32_t t = b->q_offsets_host[q]; t < b->q_offsets_host[q + 1]; ++t)
            work[t / hp.chunk] += std::min<int64_t>(L, std::max<int64_t>(0, int64_t(q_pos_host[t]) + 1));
    }
    std::vector<int32_t> order(n_chunks);
    for (int32_t c = 0; c < n_chunks; ++c) order[c] = c;
    std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t c) { return work[a] > work[c]; });

    // Events linking the streams (released once the device has passed them).
    constexpr int kEvents = 3 + 3 * kHostBufs;
    cudaEvent_t ev[kEvents];
    int made = 0;
    for (; made < kEvents; ++made)
        if (cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming) != cudaSuccess) break;
    auto release = [&]() { for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]); };
    if (made < kEvents) { release(); return DSA_ERR_CUDA; }
    cudaEvent_t e_start = ev[0], e_in = ev[1], e_out = ev[2];
    cudaEvent_t* e_q = ev + 3;                   // chunk's queries arrived in its buffer
    cudaEvent_t* e_done = ev + 3 + kHostBufs;    // chunk scored and selected: its query buffer is free
    cudaEvent_t* e_back = ev + 3 + 2 * kHostBufs;   // chunk's indices copied out: its index buffer is free
    bool ok = true;
    auto chk = [&](cudaError_t e) { ok = ok && e == cudaSuccess; };
    // the queries of the p-th chunk in processing order into buffer p % kHostBufs, once the chunk
    // kHostBufs earlier no longer reads it
    auto send_queries = [&](int32_t p) {
        const int32_t c = order[p], x = p % kHostBufs;
        if (p >= kHostBufs) chk(cudaStreamWaitEvent(si, e_done[x], 0));
        chk(cudaMemcpyAsync(hp.Q[x], static_cast<const uint8_t*>(Q) + size_t(c) * hp.chunk * qrow_bytes,
                            size_t(rows_of(c)) * qrow_bytes, cudaMemcpyHostToDevice, si));
        chk(cudaEventRecord(e_q[x], si));
    };

    // The small inputs and the keys first (after the header is cleared), then the first chunks' queries.
    chk(cudaEventRecord(e_start, st));
    chk(cudaStreamWaitEvent(si, e_start, 0));
    chk(cudaStreamWaitEvent(so, e_start, 0));
    chk(cudaMemcpyAsync(hp.q_off, b->q_offsets_host, (b->num_seqs + 1) * sizeof(int32_t), cudaMemcpyHostToDevice, si));
    chk(cudaMemcpyAsync(hp.k_off, b->k_offsets_host, (b->num_seqs + 1) * sizeof(int32_t), cudaMemcpyHostToDevice, si));
    chk(cudaMemcpyAsync(hp.q_pos, q_pos_host, size_t(nq) * sizeof(int32_t), cudaMemcpyHostToDevice, si));
    chk(cudaMemcpyAsync(hp.W, W, size_t(nq) * H * sizeof(float), cudaMemcpyHostToDevice, si));
    if (b->num_keys > 0) chk(cudaMemcpyAsync(hp.K, K, size_t(b->num_keys) * D * 2, cudaMemcpyHostToDevice, si));
    chk(cudaEventRecord(e_in, si));
    for (int32_t p = 0; p < std::min<int32_t>(kHostBufs - 1, n_chunks); ++p) send_queries(p);
    chk(cudaStreamWaitEvent(st, e_in, 0));
    if (!ok) { release(); return DSA_ERR_CUDA; }
    DSA_LAUNCH(kProfSetup, st, dense_rows_kernel<<<(nq + 255) / 256, 256, 0, st>>>(d.q_offsets, d.k_offsets, d.q_pos,
                                                                                  d.num_seqs, nq, dp.rows));
    if ((s = launched()) != DSA_OK) { release(); return s; }

    // While one chunk is scored and selected, the next chunks' queries come in and the previous
    // chunks' indices go out.
    const int64_t ld = score_ld(hi.max_k);
    for (int32_t p = 0; p < n_chunks && ok; ++p) {
        const int32_t c = order[p], r0 = c * hp.chunk, nr = rows_of(c);
        const int x = p % kHostBufs;
        if (p + kHostBufs - 1 < n_chunks) send_queries(p + kHostBufs - 1);
        chk(cudaStreamWaitEvent(st, e_q[x], 0));
        if (p >= kHostBufs) chk(cudaStreamWaitEvent(st, e_back[x], 0));   // its index buffer has been copied out
        DSA_LAUNCH(kProfSetup, st, chunk_rows_kernel<<<(nr + 255) / 256, 256, 0, st>>>(dp.rows, r0, nr, hp.rows));
        if ((s = launched()) != DSA_OK) break;
        const TcSource src{hp.Q[x], nr, hp.W + size_t(r0) * H, d.q_offsets, b->q_offsets_host, b->num_seqs};
        s = tc_score(hp.rows, nr, r0, src, H, D, hp.K, b->num_keys, d.k_offsets, ColMap{}, hi.max_k, dp.S, ld, dp.units,
                     dp.tile_base, static_cast<uint32_t*>(ws), st);
        if (s != DSA_OK) break;
        s = launch_select(hp.rows, nr, hi.max_k, k, ColMap{}, dp.S, ld, false, hp.idx[x], k, nullptr, 0, st, dp.split);
        if (s != DSA_OK) break;
        chk(cudaEventRecord(e_done[x], st));
        chk(cudaStreamWaitEvent(so, e_done[x], 0));
        chk(cudaMemcpyAsync(idx + size_t(r0) * k, hp.idx[x], size_t(nr) * k * sizeof(int32_t), cudaMemcpyDeviceToHost,
                            so));
        chk(cudaEventRecord(e_back[x], so));
    }
    // The caller's stream completes after the last index copy.
    chk(cudaEventRecord(e_out, so));
    chk(cudaStreamWaitEvent(st, e_out, 0));
    release();
    if (s != DSA_OK) return s;
    return ok ? DSA_OK : DSA_ERR_CUDA;
}

// ------------------------------------------------------------------ PIVOT
int32_t pivot_num_groups(const dsa_batch* b, int32_t group)
{
    HostInfo hi;
    if (check_batch(b, &hi) != DSA_OK || group < 1) return -1;
    return count_groups(b, group);
}

static bool pivot_args_ok(int32_t k, int32_t G, int32_t C, int32_t mode)
{
    return k >= 1 && k <= kMaxK && G >= 1 && G <= 64 && C >= k && C <= kMaxCand && (mode == 0 || mode == 1);
}

size_t pivot_group_index_workspace(const dsa_batch* b, int32_t k, int32_t G, int32_t C, int32_t mode)
{
    HostInfo hi;
    if (check_batch(b, &hi) != DSA_OK || !pivot_args_ok(k, G, C, mode)) return 0;
    PivotPlan p;
    return pivot_plan(nullptr, b, hi, k, G, C, mode, &p);
}

dsa_status pivot_group_index(const dsa_batch* b, const void* Q, const void* K, const float* W, int32_t k,
                             int32_t G, int32_t C, int32_t mode, int32_t* idx, int32_t* cand_out, void* ws,
                             size_t ws_bytes, void* stream)
{
    HostInfo hi;
    dsa_status s = check_batch(b, &hi);
    if (s != DSA_OK) return s;
    if (!pivot_args_ok(k, G, C, mode) || !select_fits(C, hi.max_k) || !select_fits(k, C)) return DSA_ERR_UNSUPPORTED;
    if ((s = check_tensors(b, Q, K, W)) != DSA_OK) return s;
    if (b->num_queries > 0 && !idx) return DSA_ERR_INVALID_ARG;
    PivotPlan p;
    if ((s = check_ws(ws, ws_bytes, pivot_plan(nullptr, b, hi, k, G, C, mode, &p))) != DSA_OK) return s;
    pivot_plan(static_cast<char*>(ws), b, hi, k, G, C, mode, &p);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((s = clear_status(ws, st)) != DSA_OK) return s;
    const int32_t ng = count_groups(b, G);
    if (ng == 0) return DSA_OK;
    const int H = b->num_heads, D = b->head_dim;
    int32_t* cand = cand_out ? cand_out : p.cand;
    const int64_t ld = score_ld(hi.max_k);
    // Reuse with no candidate list wanted, the scan's scores held at once: the group's list comes
    // from the proxy row itself (the top k + G - 1 of the top C are the top k + G - 1 of the row)
    const bool direct = mode == 0 && !cand_out && chunk_rows(ng, ld) >= ng;

    DSA_LAUNCH(kProfSetup, st, pivot_groups_kernel<<<1, 256, 0, st>>>(b->q_offsets, b->k_offsets, b->q_pos, b->num_seqs, G, ng, p.group_base,
                                           p.groups, p.proxy_rows));
    if ((s = launched()) != DSA_OK) return s;
    DSA_LAUNCH(kProfProxy, st, pivot_proxy_kernel<<<ng, 256, 0, st>>>(p.groups, static_cast<const __nv_bfloat16*>(Q), W, H, D, p.Qp, p.Wp));
    if ((s = launched()) != DSA_OK) return s;
    // Shared scan: each proxy against its prefix, top-C kept with their proxy scores.
    const std::vector<int32_t> goff = group_offsets_host(b, G);
    const TcSource src{p.Qp, ng, p.Wp, p.group_base, goff.data(), b->num_seqs};
    if (direct) return reuse_direct(b, hi, K, k, G, C, ng, src, idx, p, ws, st);
    s = tc_score_and_select(p.proxy_rows, ng, src, H, D, K, b->num_keys, b->k_offsets, ColMap{}, hi.max_k, p.S, p.units,
                            p.tile_base, static_cast<uint32_t*>(ws), C, cand, C, p.cand_score, st);
    if (s != DSA_OK) return s;
    DSA_LAUNCH(kProfSetup, st, pivot_query_rows_kernel<<<(b->num_queries + 255) / 256, 256, 0, st>>>(
        b->q_offsets, b->k_offsets, b->q_pos, b->num_seqs, b->num_queries, G, p.group_base, cand, C, nullptr,
        p.query_rows));
    if ((s = launched()) != DSA_OK) return s;
    ColMap m{};
    m.kind = kMapList;
    m.list = cand;
    m.list_ld = C;
    if (mode == 0) {
        // Reuse: rank the group's candidates by their proxy scores inside each query's prefix.  One
        // selection of the group's top k + G - 1 serves every query whose prefix keeps k of them;
        // the others (ragged positions) are ranked one by one.
        const int32_t kp = reuse_list_len(k, G, C);
        DSA_LAUNCH(kProfSetup, st, pivot_cand_rows_kernel<<<(ng + 255) / 256, 256, 0, st>>>(p.groups, ng, C, p.cand_rows));
        if ((s = launched()) != DSA_OK) return s;
        s = launch_select(p.cand_rows, ng, C, kp, identity_map(), p.cand_score, C, false, p.gsel, kp, p.gscore, kp, st);
        if (s != DSA_OK) return s;
        ReuseArgs ra{};
        ra.groups = p.groups; ra.query_rows = p.query_rows; ra.cand_rows = p.cand_rows;
        ra.gsel = p.gsel; ra.gscore = p.gscore; ra.kp = kp; ra.k = k; ra.cand = cand; ra.C = C;
        ra.idx = idx; ra.ld_idx = k; ra.fb_rows = p.fb_rows; ra.fb_count = reuse_fallback_count(ws);
        ra.status = static_cast<uint32_t*>(ws);
        const size_t smem = reuse_smem_bytes(kp);
        if ((s = set_smem(pivot_reuse_kernel, smem)) != DSA_OK) return s;
        DSA_LAUNCH(kProfSelect, st, pivot_reuse_kernel<<<ng, kReuseThreads, smem, st>>>(ra));
        if ((s = launched()) != DSA_OK) return s;
        return launch_select(p.fb_rows, b->num_queries, C, k, m, p.cand_score, C, true, idx, k, nullptr, 0, st,
                             SelectSplit{}, reuse_fallback_count(ws));
    }
    return refine_stage(b, Q, K, W, k, G, C, ng, m, idx, p, ws, st);
}

size_t pivot_refine_candidates_workspace(const dsa_batch* b, int32_t k, int32_t G, int32_t C)
{
    return pivot_group_index_workspace(b, k, G, C, 1);
}

dsa_status pivot_refine_candidates(const dsa_batch* b, const void* Q, const void* K, const float* W, int32_t k,
                                   int32_t G, int32_t C, const int32_t* cand, int32_t* idx, void* ws,
                                   size_t ws_bytes, void* stream)
{
    HostInfo hi;
    dsa_status s = check_batch(b, &hi);
    if (s != DSA_OK) return s;
    if (!pivot_args_ok(k, G, C, 1) || !select_fits(k, C)) return DSA_ERR_UNSUPPORTED;
    if ((s = check_tensors(b, Q, K, W)) != DSA_OK) return s;
    if (b->num_queries > 0 && (!idx || !cand)) return DSA_ERR_INVALID_ARG;
    PivotPlan p;
    if ((s = check_ws(ws, ws_bytes, pivot_plan(nullptr, b, hi, k, G, C, 1, &p))) != DSA_OK) return s;
    pivot_plan(static_cast<char*>(ws), b, hi, k, G, C, 1, &p);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((s = clear_status(ws, st)) != DSA_OK) return s;
    const int32_t ng = count_groups(b, G);
    if (ng == 0) return DSA_OK;
    DSA_LAUNCH(kProfSetup, st, pivot_groups_kernel<<<1, 256, 0, st>>>(b->q_offsets, b->k_offsets, b->q_pos, b->num_seqs, G,
                                                                       ng, p.group_base, p.groups, p.proxy_rows));
    if ((s = launched()) != DSA_OK) return s;
    // the caller's lists: usable lengths (the proxy row array is free scratch here)
    int32_t* cand_len = reinterpret_cast<int32_t*>(p.proxy_rows);
    DSA_LAUNCH(kProfSetup, st, pivot_check_cand_kernel<<<(ng + 7) / 8, 256, 0, st>>>(cand, C, p.groups, ng, b->k_offsets,
                                                                                      cand_len, static_cast<uint32_t*>(ws)));
    if ((s = launched()) != DSA_OK) return s;
    DSA_LAUNCH(kProfSetup, st, pivot_query_rows_kernel<<<(b->num_queries + 255) / 256, 256, 0, st>>>(
        b->q_offsets, b->k_offsets, b->q_pos, b->num_seqs, b->num_queries, G, p.group_base, cand, C, cand_len,
        p.query_rows));
    if ((s = launched()) != DSA_OK) return s;
    ColMap m{};
    m.kind = kMapList;
    m.list = cand;
    m.list_ld = C;
    return refine_stage(b, Q, K, W, k, G, C, ng, m, idx, p, ws, st);
}

// ------------------------------------------------------------------- HISA
static bool hisa_args_ok(int32_t k, int32_t B, int32_t keep)
{
    return k >= 1 && k <= kMaxK && (B == 64 || B == 128 || B == 256) && keep >= 1 && keep <= 256;
}

int64_t hisa_num_blocks(const dsa_batch* b, int32_t B)
{
    HostInfo hi;
    if (check_batch(b, &hi) != DSA_OK || B < 1) return -1;
    int64_t n = 0;
    for (int i = 0; i < b->num_seqs; ++i) n += (b->k_offsets_host[i + 1] - b->k_offsets_host[i] + B - 1) / B;
    return n;
}

dsa_status hisa_pool_keys(const dsa_batch* b, const void* K, int32_t B, float* pooled, void* stream)
{
    HostInfo hi;
    dsa_status s = check_batch(b, &hi);
    if (s != DSA_OK) return s;
    if (!(B == 64 || B == 128 || B == 256)) return DSA_ERR_UNSUPPORTED;
    const int64_t nb = hisa_num_blocks(b, B);
    if (nb == 0) return DSA_OK;
    if (!K || !pooled || (reinterpret_cast<uintptr_t>(K) & 15) || (reinterpret_cast<uintptr_t>(pooled) & 15))
        return DSA_ERR_INVALID_ARG;
    if (nb > INT32_MAX) return DSA_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DSA_LAUNCH(kProfPool, st, hisa_pool_kernel<<<(unsigned)nb, b->head_dim, 0, st>>>(static_cast<const __nv_bfloat16*>(K), b->k_offsets,
                                                          b->num_seqs, B, b->head_dim, pooled));
    return launched();
}

size_t hisa_index_workspace(const dsa_batch* b, int32_t k, int32_t B, int32_t keep)
{
    HostInfo hi;
    if (check_batch(b, &hi) != DSA_OK || !hisa_args_ok(k, B, keep)) return 0;
    HisaPlan p;
    return hisa_plan(nullptr, b, hi, k, B, keep, &p);
}

dsa_status hisa_index(const dsa_batch* b, const void* Q, const void* K, const float* W, const float* pooled,
                      int32_t k, int32_t B, int32_t keep, int32_t* idx, int32_t* kept_out, void* ws, size_t ws_bytes,
                      void* stream)
{
    HostInfo hi;
    dsa_status s = check_batch(b, &hi);
    if (s != DSA_OK) return s;
    if (!hisa_args_ok(k, B, keep) || !select_fits(keep, std::max(0, (hi.max_k + B - 1) / B - 2)))
        return DSA_ERR_UNSUPPORTED;
    if ((s = check_tensors(b, Q, K, W)) != DSA_OK) return s;
    if (b->num_queries > 0 && (!idx || !pooled)) return DSA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(pooled) & 15) return DSA_ERR_INVALID_ARG;
    HisaPlan p;
    if ((s = check_ws(ws, ws_bytes, hisa_plan(nullptr, b, hi, k, B, keep, &p))) != DSA_OK) return s;
    hisa_plan(static_cast<char*>(ws), b, hi, k, B, keep, &p);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int32_t nq = b->num_queries;
    if (nq == 0) return clear_status(ws, st);
    g_status = static_cast<uint32_t*>(ws);   // hisa_setup_kernel clears the header
    const int H = b->num_heads, D = b->head_dim;
    int32_t* kept = kept_out ? kept_out : p.kept;
    if (p.planes) return hisa_one_pass(b, hi, Q, K, W, pooled, k, B, keep, idx, kept, p, ws, st);
    const unsigned g = (nq + 255) / 256;

    DSA_LAUNCH(kProfSetup, st, hisa_setup_kernel<<<(nq + 256) / 256, 256, 0, st>>>(b->q_offsets, b->k_offsets, b->q_pos,
                                                    b->num_seqs, nq, B, p.block_base, p.block_rows, p.query_off,
                                                    static_cast<uint32_t*>(ws), (int32_t)(kHeaderBytes / 4)));
    if ((s = launched()) != DSA_OK) return s;
    // Coarse stage: middle blocks scored on their pooled keys, top `keep` kept.
    const int32_t max_mid = std::max(0, (hi.max_k + B - 1) / B - 2);
    s = score_and_select<float>(p.block_rows, nq, max_mid, identity_map(1), Q, W, H, D, pooled, p.block_base, p.S,
                                keep, p.mid, keep, nullptr, st);
    if (s != DSA_OK) return s;
    // Fine stage: the indexer over the tokens of the kept blocks.
    ColMap m{};
    m.kind = kMapBlocks;
    m.block = B;
    m.list = kept;
    m.list_ld = keep + 2;
    const std::vector<int32_t> qoff = iota_host(nq);
    const TcSource src{Q, nq, W, p.query_off, qoff.data(), nq};
    const int32_t tok_cols = (keep + 2) * B;
    const int64_t ld_tok = score_ld(tok_cols);
    if (chunk_rows(nq, ld_tok) >= nq) {
        // one scoring launch: kept blocks, token rows and its units in one kernel (a warp per query)
        const int32_t splits = tc_splits(tc_count_tiles(qoff.data(), nq, 0, nq, tc_tile_rows(H)), tok_cols);
        DSA_LAUNCH(kProfSetup, st, launch_pdl(latency_bound(nq), hisa_kept_units_kernel, (nq + 7) / 8, 256, 0, st,
                                              p.block_rows, p.mid, keep, b->q_pos, b->k_offsets, nq, B, splits, kept,
                                              p.token_rows, p.units));
        if ((s = launched()) != DSA_OK) return s;
        s = tc_score(p.token_rows, nq, 0, src, H, D, K, b->num_keys, b->k_offsets, m, tok_cols, p.S, ld_tok, p.units,
                     p.tile_base, static_cast<uint32_t*>(ws), st, TcOpts{true});
        if (s != DSA_OK) return s;
        return launch_select(p.token_rows, nq, tok_cols, k, m, p.S, ld_tok, false, idx, k, nullptr, 0, st, p.split);
    }
    DSA_LAUNCH(kProfSetup, st, hisa_kept_kernel<<<g, 256, 0, st>>>(p.block_rows, p.mid, keep, b->q_pos, b->k_offsets, nq, B, kept,
                                        p.token_rows));
    if ((s = launched()) != DSA_OK) return s;
    return tc_score_and_select(p.token_rows, nq, src, H, D, K, b->num_keys, b->k_offsets, m, tok_cols, p.S,
                               p.units, p.tile_base, static_cast<uint32_t*>(ws), k, idx, k, nullptr, st, p.split);
}

// ---------------------------------------------------------------- profiling
void dsa_profile_enable(int32_t on)
{
    g_prof_on.store(on != 0);
}

uint64_t dsa_launch_count(void)
{
    return g_launches.load();
}

const char* dsa_profile_kind_name(int32_t kind)
{
    return (kind >= 0 && kind < kProfKinds) ? kProfNames[kind] : nullptr;
}

int32_t dsa_profile_read(float* ms, int32_t* launches, int32_t cap)
{
    std::vector<ProfRec> recs;
    {
        std::lock_guard<std::mutex> lk(g_prof_mu);
        recs.swap(g_prof);
    }
    for (int32_t k = 0; k < cap && k < kProfKinds; ++k) {
        if (ms) ms[k] = 0.f;
        if (launches) launches[k] = 0;
    }
    int32_t status = kProfKinds;
    for (const ProfRec& r : recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
            status = -1;
        if (r.kind < cap) {
            if (ms) ms[r.kind] += t;
            if (launches) launches[r.kind] += 1;
        }
        cudaEventDestroy(r.start);
        cudaEventDestroy(r.stop);
    }
    return status;
}

// ------------------------------------------------------------ device check
dsa_status dsa_selftest_wait_timeout(uint32_t limit_us, void* ws, size_t ws_bytes, void* stream)
{
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) || ws_bytes < kStatusBytes) return DSA_ERR_INVALID_ARG;
    if (limit_us < 1 || limit_us > 1000000) return DSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, kStatusBytes, st) != cudaSuccess) return DSA_ERR_CUDA;
    DSA_LAUNCH(kProfSetup, st, selftest_wait_kernel<<<1, 32, 0, st>>>(static_cast<uint32_t*>(ws),
                                                                      uint64_t(limit_us) * 1000u));
    return launched();
}

dsa_status dsa_device_check(void* ws, void* stream, uint32_t* detail)
{
    if (!ws) return DSA_ERR_INVALID_ARG;
    uint32_t h[2] = {0, 0};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(h, ws, sizeof h, cudaMemcpyDeviceToHost, st) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
    if (h[0] == 0) return DSA_OK;
    if (detail) *detail = h[0];
    if (cudaMemsetAsync(ws, 0, 8, st) != cudaSuccess) return DSA_ERR_CUDA;
    return DSA_ERR_DEVICE_CHECK;
}

}  // extern "C"

// =====================================================================
// Allocation-free variant of dsa_index_topk.
//
// Some callers cannot call cudaMalloc at all: for example an inference
// runtime's custom-op callback that is handed no allocator and must not
// allocate while it runs, or a latency-critical loop that is not allowed to
// touch the device allocator.  For them the workspace of dsa_index_topk lives
// in this file-scope device array instead of caller memory.  Every GPU that
// loads the library holds it (kStaticScratchBytes) until the process exits.
namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;   // 8 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch in the current device's context.  In host code the array's
// name is only a host-side stand-in, so the address is looked up with cudaGetSymbolAddress (with
// that device current) on every call: a cached address would go stale once the context is
// destroyed and made again (cudaDeviceReset, or the primary context released and retained),
// which loads the module again, possibly elsewhere.  The lookup allocates nothing.
dsa_status static_scratch(void** out)
{
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
    *out = p;
    return DSA_OK;
}

}  // namespace

extern "C" size_t dsa_index_topk_static_capacity(void) { return kStaticScratchBytes; }

extern "C" dsa_status dsa_index_topk_static(const dsa_batch* b, const void* Q, const void* K, const float* W,
                                            int32_t k, int32_t* idx, float* scores, void* stream)
{
    HostInfo hi;
    dsa_status s = check_batch(b, &hi);
    if (s != DSA_OK) return s;
    if (k < 1 || k > kMaxK || !select_fits(k, hi.max_k)) return DSA_ERR_UNSUPPORTED;
    DensePlan p;
    if (dense_plan(nullptr, b, hi, k, &p) > kStaticScratchBytes) return DSA_ERR_WORKSPACE;
    void* ws = nullptr;
    if ((s = static_scratch(&ws)) != DSA_OK) return s;
    // dsa_index_topk clears the workspace header (status word, select counters) at the start of
    // every call; nothing else must start at zero.
    return dsa_index_topk(b, Q, K, W, k, idx, scores, ws, kStaticScratchBytes, stream);
}
