// Shared device-side definitions of libdsaidx: row descriptors, column maps,
// the order-preserving score key and the workspace status word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dsa {

// ---------------------------------------------------------------- status
// The first 256 bytes of every workspace.  word 0: first error code recorded
// by any kernel (0 = none); word 1: detail (where it happened).
constexpr size_t kStatusBytes = 256;
enum : uint32_t {
    kErrNone = 0,
    kErrWaitTimeout = 1,   // a bounded wait on an mbarrier ran out
    kErrBadRow = 2,        // a row descriptor points outside its buffers
    kErrBadIndex = 4,      // (checked builds) an index computed on the device fell outside its buffer
};

__device__ __forceinline__ void record_error(uint32_t* status, uint32_t code, uint32_t detail)
{
    if (!status) return;
    if (atomicCAS(status, 0u, code) == 0u)
        status[1] = detail;
}

// Checked builds (compiled with -DDSA_DEVICE_CHECKS=1): DSA_CHECK(ok, status, where) is `ok`, and a
// false `ok` records kErrBadIndex with detail `where` in the status word, so the caller can skip the
// access it guards.  Otherwise it is `true` and costs nothing.  Every guarded index is in range by
// construction; the checks exist to catch a broken invariant (a gathered key row, a candidate
// position, a bitmap word, an output slot) without a memory fault.
#ifndef DSA_DEVICE_CHECKS
#define DSA_DEVICE_CHECKS 0
#endif
__device__ __forceinline__ bool check_index(bool ok, uint32_t* status, uint32_t where)
{
    if (!ok) record_error(status, kErrBadIndex, where);
    return ok;
}
#if DSA_DEVICE_CHECKS
#define DSA_CHECK(ok, status, where) (::dsa::check_index((ok), (status), (where)))
#else
#define DSA_CHECK(ok, status, where) (true)
#endif

// -------------------------------------------------------- score ordering
// Order-preserving map of an fp32 score to uint32: a larger score gives a
// larger key, -0 maps like +0 (the ranking treats them as equal).
__device__ __forceinline__ uint32_t score_key(float v)
{
    uint32_t u = __float_as_uint(v);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint32_t k)
{
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// ------------------------------------------------------- rows and columns
// A "row" is one ranking problem: one query (or proxy) against an ordered
// set of candidate keys of its sequence.  Column c of the row is a key
// index; the map from columns to keys is increasing, so "lower column"
// and "lower key index" break ties the same way.
struct RowDesc {
    int32_t qrow;    // row of the query arrays (Q/W, or the proxy arrays)
    int32_t seq;     // sequence
    int32_t ncols;   // eligible columns [0, ncols)
    int32_t list;    // row of the map's list (kMapList / kMapBlocks)
};

enum MapKind : int32_t {
    kMapIdentity = 0,   // key = col + offset
    kMapList = 1,       // key = list[row.list * list_ld + col]
    kMapBlocks = 2,     // key = list[row.list * list_ld + col / block] * block + col % block
};

struct ColMap {
    int32_t kind;
    int32_t offset;
    int32_t block;
    int32_t pad_;
    const int32_t* list;
    int64_t list_ld;
};

__device__ __forceinline__ int32_t map_col(const ColMap& m, const RowDesc& r, int32_t col)
{
    if (m.kind == kMapIdentity) return col + m.offset;
    const int32_t* l = m.list + (int64_t)r.list * m.list_ld;
    if (m.kind == kMapList) return l[col];
    return l[col / m.block] * m.block + col % m.block;
}

// Eligible keys of a query: s <= pos, s < L.
__device__ __forceinline__ int32_t eligible_count(int32_t pos, int32_t L)
{
    if (pos < 0) return 0;
    return pos + 1 < L ? pos + 1 : L;
}

__device__ __forceinline__ int32_t find_seq(const int32_t* offsets, int32_t n_seqs, int32_t row)
{
    int32_t lo = 0, hi = n_seqs - 1;
    while (lo < hi) {
        int32_t mid = (lo + hi + 1) >> 1;
        if (offsets[mid] <= row) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// One work unit of the tensor-core scoring kernel: consecutive query rows of one segment and a
// range of its key tiles, with what the TMA producer needs to start at once.
struct TcUnit {
    int32_t row0;    // first row of the unit in the launch's row array
    int32_t nrows;   // consecutive rows of one segment
    int32_t kt0;     // key tiles [kt0, kt1) of 128 keys, segment-local
    int32_t kt1;
    int32_t qrow;    // query row (Q / W) of row0
    int32_t krow0;   // key row of the segment's key 0: k_base[seq]
    int32_t pad_[2];
};

// Programmatic dependent launch: a kernel launched with programmatic stream serialization may
// start while its predecessor still runs; grid_dep_wait() returns once the predecessor grid has
// completed and its memory is visible (at once for a kernel launched without it), and
// grid_dep_launch() lets the successor's CTAs be scheduled once every CTA of this grid has
// called it or exited.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t lanemask_lt()
{
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace dsa
