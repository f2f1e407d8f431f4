// common.cuh -- shared device helpers of libeagleattn.
//
// Visibility of block-0 keys is expressed per query row as one interval of
// local key indices [lo_t, hi_t]: a key s is visible to row t iff
// lo_t <= s <= hi_t.  The interval is the intersection of
//   - the row's packed document [cu[d], cu[d+1]) (NeMo AutoModel
//     "eagle.ulysses_attention", _block0_forward, parameter cu_seqlens),
//   - the causal half-line k_pos <= q_pos with global positions
//     q_pos = q_pos_offset + t, k_pos = k_pos_offset + s ("target_cp",
//     attach_cp_kv_gather_hooks),
//   - the key range [0, Tk).
// Both ends are non-decreasing in t, which is what makes tile skipping and
// the backward's row ranges cheap.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/eagleattn.h"

namespace eagle {

// Sticky device status word of this library (one per device / context).
__device__ int g_status;

__device__ __forceinline__ void raise_status(int code) { atomicCAS(&g_status, 0, code); }
__device__ __forceinline__ bool status_bad() { return *(volatile int *)&g_status != 0; }

struct MaskDesc {
    const int32_t *cu;  // device cu_seqlens or nullptr
    int num_docs;
    int64_t q_off, k_off;
    int causal;
    int Tq, Tk;
};

// The mask functions below also compile for the host, where a test checks them
// against a brute-force visibility count.
#ifdef __CUDA_ARCH__
#define EAGLE_LDG(p) __ldg(p)
#else
#define EAGLE_LDG(p) (*(p))
#endif
#define EAGLE_HD __host__ __device__ __forceinline__

// Document holding global position pos (binary search); -1 if none.
EAGLE_HD int find_doc(const int32_t *cu, int nd, int64_t pos) {
    if (pos < 0 || pos >= (int64_t)EAGLE_LDG(cu + nd)) return -1;
    int lo = 0, hi = nd - 1;  // invariant: cu[lo] <= pos < cu[hi+1]
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((int64_t)EAGLE_LDG(cu + mid) <= pos) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Visible local key interval [lo, hi] of query row t.  Returns the row's
// class: 0 = non-empty interval; -1 = empty because everything the row may
// see lies before key 0; +1 = empty because it lies past key Tk-1.  The class
// is non-decreasing in t (a prefix of -1, then 0, then a suffix of +1) and, on
// the class-0 rows, lo and hi are non-decreasing in t.
EAGLE_HD int row_interval(const MaskDesc &m, int t, int &lo, int &hi) {
    int64_t qp = m.q_off + t;
    int64_t glo = INT64_MIN / 4, ghi = INT64_MAX / 4;
    if (m.cu) {
        int d = find_doc(m.cu, m.num_docs, qp);
        if (d < 0) { lo = 0; hi = -1; return qp < 0 ? -1 : 1; }
        glo = EAGLE_LDG(m.cu + d);
        ghi = (int64_t)EAGLE_LDG(m.cu + d + 1) - 1;
    }
    if (m.causal && qp < ghi) ghi = qp;
    int64_t l = glo - m.k_off, h = ghi - m.k_off;
    if (h < 0) { lo = 0; hi = -1; return -1; }
    if (l > m.Tk - 1) { lo = 0; hi = -1; return 1; }
    lo = (int)(l < 0 ? 0 : l);
    hi = (int)(h > m.Tk - 1 ? m.Tk - 1 : h);
    return 0;
}

// [lo, hi] (global positions) intersected with [0, n): as local indices [a, b]
// (b < a when empty).
EAGLE_HD void clip_range(int64_t lo, int64_t hi, int64_t off, int n, int &a, int &b) {
    lo -= off;
    hi -= off;
    if (lo < 0) lo = 0;
    if (hi > n - 1) hi = n - 1;
    if (lo > hi) { a = 0; b = -1; return; }
    a = (int)lo;
    b = (int)hi;
}

// Key range [kbeg, kend] seen by query rows [t0, t1] (t0 <= t1); kend < kbeg if
// none.  A row sees from its document's start (from everything, without
// documents) to its own position (causal) or its document's end, so the rows of a
// range see one interval: from the first row's document start to the last row's
// position or document end.
EAGLE_HD void rows_key_range(const MaskDesc &m, int t0, int t1, int &kbeg, int &kend) {
    if (t1 < t0) { kbeg = 0; kend = -1; return; }
    int64_t a = m.q_off + t0, c = m.q_off + t1;
    int64_t glo = INT64_MIN / 4, ghi = m.causal ? c : INT64_MAX / 4;
    if (m.cu) {
        // rows outside every document see nothing
        const int64_t end = EAGLE_LDG(m.cu + m.num_docs);
        if (a < 0) a = 0;
        if (c > end - 1) c = end - 1;
        if (a > c) { kbeg = 0; kend = -1; return; }
        glo = EAGLE_LDG(m.cu + find_doc(m.cu, m.num_docs, a));
        ghi = m.causal ? c : (int64_t)EAGLE_LDG(m.cu + find_doc(m.cu, m.num_docs, c) + 1) - 1;
    }
    clip_range(glo, ghi, m.k_off, m.Tk, kbeg, kend);
}

// Query rows [tbeg, tend] that see a key in [k0, k1] (0 <= k0 <= k1 < Tk); tend <
// tbeg if none.  By the same argument, from the first key's position (causal) or
// document start to the last key's document end.
EAGLE_HD void keys_row_range(const MaskDesc &m, int k0, int k1, int &tbeg, int &tend) {
    if (k1 < k0) { tbeg = 0; tend = -1; return; }
    int64_t a = m.k_off + k0, c = m.k_off + k1;
    int64_t glo = m.causal ? a : INT64_MIN / 4, ghi = INT64_MAX / 4;
    if (m.cu) {
        const int64_t end = EAGLE_LDG(m.cu + m.num_docs);
        if (a < 0) a = 0;
        if (c > end - 1) c = end - 1;
        if (a > c) { tbeg = 0; tend = -1; return; }
        glo = m.causal ? a : (int64_t)EAGLE_LDG(m.cu + find_doc(m.cu, m.num_docs, a));
        ghi = (int64_t)EAGLE_LDG(m.cu + find_doc(m.cu, m.num_docs, c) + 1) - 1;
    }
    clip_range(glo, ghi, m.q_off, m.Tq, tbeg, tend);
}

// Query rows [ta, tb] that see local key s (empty, tb < ta, for s outside [0, Tk)).
EAGLE_HD void key_rows(const MaskDesc &m, int s, int &ta, int &tb) {
    if (s < 0 || s >= m.Tk) { ta = 0; tb = -1; return; }
    keys_row_range(m, s, s, ta, tb);
}

// Block order of the tile kernels.  Blocks start in increasing linear index, so
// the tile index (0 = the tile with the most steps under the causal masks) is made
// the slow index within groups of HEAVY_GROUP (batch, head) pairs: a group's
// heaviest tiles start first and its lightest end it, which keeps the last wave
// short, while only the group's pairs share L2.  lin = the block's linear index
// over a grid of ntiles x npairs blocks; returns its tile and pair (b * H + h).
constexpr int HEAVY_GROUP = 8;
EAGLE_HD void heavy_first(int lin, int ntiles, int npairs, int &tile, int &pair) {
    const int first = lin / (HEAVY_GROUP * ntiles) * HEAVY_GROUP;  // the group's first pair
    const int gs = npairs - first < HEAVY_GROUP ? npairs - first : HEAVY_GROUP;
    const int idx = lin - first * ntiles;
    tile = idx / gs;
    pair = first + idx % gs;
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Query segment i of a q_tiles list: rows [t0, t0 + n).  False (and the CTA or
// warp skips it) when the entry is out of range: t0 outside [0, Tq), n outside
// 1 .. 128, t0 + n past Tq, or, for a list without row counts, t0 not a
// multiple of 128.
__device__ __forceinline__ bool q_segment(const int32_t *starts, const int32_t *rows, int i,
                                          int Tq, int &t0, int &n) {
    t0 = __ldg(starts + i);
    if (t0 < 0 || t0 >= Tq) return false;
    if (rows) {
        n = __ldg(rows + i);
        return n >= 1 && n <= 128 && n <= Tq - t0;
    }
    n = Tq - t0 < 128 ? Tq - t0 : 128;
    return (t0 & 127) == 0;
}

// Kernel-side view of the problem (strides in elements).
struct Problem {
    int B, Tq, Tk, H, D, NB;
    float scale;
    int64_t q_sb, q_st;             // q, out, grad_out, dq
    int64_t kv_sb, kv_sblk, kv_st;  // cache_k, cache_v, dk, dv
    int grad_accum;                 // backward: dq/dk/dv are fp32 and the call adds into them
    const int32_t *q_tiles;         // the query tiles / segments to compute, or null (all)
    const int32_t *q_tile_rows;     // rows of each q_tiles entry, or null (128-row tiles)
    int num_q_tiles;
    MaskDesc mask;
};

}  // namespace eagle
