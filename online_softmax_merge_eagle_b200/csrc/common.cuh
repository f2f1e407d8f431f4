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

// Document holding global position pos (binary search); -1 if none.
__device__ __forceinline__ int find_doc(const int32_t *cu, int nd, int64_t pos) {
    if (pos < 0 || pos >= (int64_t)__ldg(cu + nd)) return -1;
    int lo = 0, hi = nd - 1;  // invariant: cu[lo] <= pos < cu[hi+1]
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((int64_t)__ldg(cu + mid) <= pos) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Visible local key interval [lo, hi] of query row t.  Returns the row's
// class: 0 = non-empty interval; -1 = empty because everything the row may
// see lies before key 0; +1 = empty because it lies past key Tk-1.  The class
// is non-decreasing in t (a prefix of -1, then 0, then a suffix of +1) and, on
// the class-0 rows, lo and hi are non-decreasing in t.
__device__ __forceinline__ int row_interval(const MaskDesc &m, int t, int &lo, int &hi) {
    int64_t qp = m.q_off + t;
    int64_t glo = INT64_MIN / 4, ghi = INT64_MAX / 4;
    if (m.cu) {
        int d = find_doc(m.cu, m.num_docs, qp);
        if (d < 0) { lo = 0; hi = -1; return qp < 0 ? -1 : 1; }
        glo = __ldg(m.cu + d);
        ghi = (int64_t)__ldg(m.cu + d + 1) - 1;
    }
    if (m.causal && qp < ghi) ghi = qp;
    int64_t l = glo - m.k_off, h = ghi - m.k_off;
    if (h < 0) { lo = 0; hi = -1; return -1; }
    if (l > m.Tk - 1) { lo = 0; hi = -1; return 1; }
    lo = (int)(l < 0 ? 0 : l);
    hi = (int)(h > m.Tk - 1 ? m.Tk - 1 : h);
    return 0;
}

// Key range [kbeg, kend] touched by query rows [t0, t1]; kend < kbeg if none.
__device__ __forceinline__ void rows_key_range(const MaskDesc &m, int t0, int t1, int &kbeg,
                                               int &kend) {
    int l, h;
    // ta = first row in [t0, t1] of class >= 0
    int a = t0, b = t1 + 1;
    while (a < b) {
        int mid = (a + b) >> 1;
        if (row_interval(m, mid, l, h) >= 0) b = mid; else a = mid + 1;
    }
    int ta = a;
    // tb = last row in [t0, t1] of class <= 0
    a = t0 - 1; b = t1;
    while (a < b) {
        int mid = (a + b + 1) >> 1;
        if (row_interval(m, mid, l, h) <= 0) a = mid; else b = mid - 1;
    }
    int tb = a;
    if (ta > tb || ta > t1 || tb < t0) { kbeg = 0; kend = -1; return; }
    int c0 = row_interval(m, ta, l, h);
    kbeg = l;
    int c1 = row_interval(m, tb, l, h);
    kend = h;
    if (c0 != 0 || c1 != 0) { kbeg = 0; kend = -1; }
}

// Query rows whose interval meets keys [k0, k1]: the contiguous range
// [tbeg, tend] (tend < tbeg if none).
__device__ __forceinline__ void keys_row_range(const MaskDesc &m, int k0, int k1, int &tbeg,
                                               int &tend) {
    int l, h;
    // first t with class +1, or class 0 and hi_t >= k0  (a monotone predicate)
    int a = 0, b = m.Tq;
    while (a < b) {
        int mid = (a + b) >> 1;
        int c = row_interval(m, mid, l, h);
        if (c > 0 || (c == 0 && h >= k0)) b = mid; else a = mid + 1;
    }
    tbeg = a;
    // last t with class -1, or class 0 and lo_t <= k1
    a = -1; b = m.Tq - 1;
    while (a < b) {
        int mid = (a + b + 1) >> 1;
        int c = row_interval(m, mid, l, h);
        if (c < 0 || (c == 0 && l <= k1)) a = mid; else b = mid - 1;
    }
    tend = a;
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
