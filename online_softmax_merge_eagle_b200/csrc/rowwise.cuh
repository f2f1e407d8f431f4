// rowwise.cuh -- memory-bound kernels that work one attention row at a time:
//   merge_kernel          (out, lse) <- (out, lse) (+) (block_out, block_lse)
//   merge_diag_kernel     fold the diagonal blocks i >= 1 into (out, lse)
//   finalize_kernel       fp32 -> output dtype
//   bwd_prep_kernel       D_t = dO_t . O_t, zero the dQ accumulator
//   bwd_diag_kernel       diagonal dq/dk/dv in closed form + dq write-out
//   bwd_rows_kernel       D_t, diagonal dk/dv and sum_i dz_i k_i for the tensor-core backward
//   dq_finalize_kernel    dq = scale * the fp32 dQ accumulator (five-product backward)
//   wait_timeout_selftest_kernel   the bounded pipeline wait giving up (self-test)
// Rows are (b, t, h) triples; row r of a contiguous [B, T, H, D] tensor starts
// at r * D, and its lse sits at (b * H + h) * T + t.
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace eagle {

// Online-softmax merge of one row pair; la/lb may be -inf (empty part).
// NeMo AutoModel "eagle.ring_attention", _update_out_and_lse: the merged lse
// is log(e^la + e^lb) and the weights are sigmoid(la - lb), sigmoid(lb - la).
struct MergeW {
    float wa, wb, l;
};
__device__ __forceinline__ MergeW merge_weights(float la, float lb) {
    MergeW w;
    if (lb == -INFINITY) {
        w.wa = la == -INFINITY ? 0.f : 1.f;
        w.wb = 0.f;
        w.l = la;
    } else if (la == -INFINITY) {
        w.wa = 0.f;
        w.wb = 1.f;
        w.l = lb;
    } else {
        float mx = fmaxf(la, lb), d = -fabsf(la - lb);
        float e = expf(d);                 // in (0, 1]
        w.l = mx + log1pf(e);
        float s = 1.f / (1.f + e);         // weight of the larger side
        float bigw = s, smallw = e * s;
        if (la >= lb) { w.wa = bigw; w.wb = smallw; } else { w.wa = smallw; w.wb = bigw; }
    }
    return w;
}

template <typename TB> struct Vec4;
template <> struct Vec4<float> {
    static __device__ __forceinline__ float4 load(const float *p) {
        return __ldcs(reinterpret_cast<const float4 *>(p));
    }
};
template <> struct Vec4<__nv_bfloat16> {
    static __device__ __forceinline__ float4 load(const __nv_bfloat16 *p) {
        uint2 u = __ldcs(reinterpret_cast<const uint2 *>(p));
        float4 f;
        f.x = __uint_as_float(u.x << 16);
        f.y = __uint_as_float(u.x & 0xffff0000u);
        f.z = __uint_as_float(u.y << 16);
        f.w = __uint_as_float(u.y & 0xffff0000u);
        return f;
    }
};

constexpr int MERGE_THREADS = 128;  // 4 warps
constexpr int MERGE_TW = 32;        // consecutive t per warp (one lse vector load)
constexpr int MERGE_U = 2;          // rows per lane in flight

// One warp per 32 consecutive t of one (b, h): the lse pair of those rows is
// one coalesced load, and each row's D floats are read by D/4 lanes as float4
// (32 / (D/4) rows per warp instruction), MERGE_U rows in flight per lane.
// Grid: (H, ceil(T / (4 * 32)), B), the head fastest: the rows of all heads of a
// t range are adjacent in memory, so the blocks in flight together read whole
// DRAM pages instead of one head's slice of many.  Twelve blocks per SM (40
// registers): more rows in flight per SM than the nine the unbounded form fits.
template <typename TB, int D4>
__global__ void __launch_bounds__(MERGE_THREADS, 12) merge_kernel(float *__restrict__ out,
                                                             float *__restrict__ lse,
                                                             const TB *__restrict__ bout,
                                                             const float *__restrict__ blse,
                                                             int T, int H, int init) {
    constexpr int RPI = 32 / D4;  // rows per warp instruction
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h = blockIdx.x, b = blockIdx.z;
    const int t0 = (blockIdx.y * (MERGE_THREADS / 32) + warp) * MERGE_TW;
    if (t0 >= T) return;
    const int64_t lbase = ((int64_t)b * H + h) * T;
    const bool lv = t0 + lane < T;
    const float lb_v = lv ? __ldg(blse + lbase + t0 + lane) : 0.f;
    const float la_v = (lv && !init) ? lse[lbase + t0 + lane] : 0.f;
    float lnew = 0.f;  // the new lse of row t0 + lane
    const int sub = lane / D4, c = lane % D4;
#pragma unroll 1
    for (int r0 = 0; r0 < MERGE_TW; r0 += RPI * MERGE_U) {
        float4 o[MERGE_U], bo[MERGE_U];
        bool ok[MERGE_U];
        int64_t off[MERGE_U];
#pragma unroll
        for (int u = 0; u < MERGE_U; ++u) {
            const int r = r0 + u * RPI + sub;
            const int t = t0 + r;
            ok[u] = t < T;
            off[u] = (((int64_t)b * T + t) * H + h) * (D4 * 4) + c * 4;
            if (ok[u]) {
                bo[u] = Vec4<TB>::load(bout + off[u]);
                if (!init) o[u] = __ldcs(reinterpret_cast<const float4 *>(out + off[u]));
            }
        }
#pragma unroll
        for (int u = 0; u < MERGE_U; ++u) {
            const int r = r0 + u * RPI + sub;
            const float la = __shfl_sync(0xffffffffu, la_v, r);
            const float lb = __shfl_sync(0xffffffffu, lb_v, r);
            float4 res;
            float l;
            if (init) {
                res = bo[u];
                l = lb;
            } else {
                const MergeW w = merge_weights(la, lb);
                res.x = w.wa * o[u].x + w.wb * bo[u].x;
                res.y = w.wa * o[u].y + w.wb * bo[u].y;
                res.z = w.wa * o[u].z + w.wb * bo[u].z;
                res.w = w.wa * o[u].w + w.wb * bo[u].w;
                l = w.l;
            }
            if (ok[u]) __stcs(reinterpret_cast<float4 *>(out + off[u]), res);
            // row r0 + u*RPI + q was merged by lane group q; lane (row - t0) keeps its lse
#pragma unroll
            for (int q = 0; q < RPI; ++q) {
                const float lq = __shfl_sync(0xffffffffu, l, q * D4);
                if (lane == r0 + u * RPI + q) lnew = lq;
            }
        }
    }
    if (lv) lse[lbase + t0 + lane] = lnew;
}

// E = D / 32 elements per lane.
template <typename T, int E> struct RowIO;
template <typename T> struct RowIO<T, 1> {
    static __device__ __forceinline__ void load(const T *p, float *f) { f[0] = to_f32<T>(p[0]); }
    static __device__ __forceinline__ void store(T *p, const float *f) { p[0] = from_f32<T>(f[0]); }
};
template <typename T> struct RowIO<T, 2> {
    static __device__ __forceinline__ void load(const T *p, float *f) {
        f[0] = to_f32<T>(p[0]);
        f[1] = to_f32<T>(p[1]);
    }
    static __device__ __forceinline__ void store(T *p, const float *f) {
        p[0] = from_f32<T>(f[0]);
        p[1] = from_f32<T>(f[1]);
    }
};
template <> struct RowIO<__nv_bfloat16, 4> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float *f) {
        uint2 u = *reinterpret_cast<const uint2 *>(p);
        f[0] = __uint_as_float(u.x << 16);
        f[1] = __uint_as_float(u.x & 0xffff0000u);
        f[2] = __uint_as_float(u.y << 16);
        f[3] = __uint_as_float(u.y & 0xffff0000u);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float *f) {
        __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]);
        __nv_bfloat162 b = __floats2bfloat162_rn(f[2], f[3]);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t *>(&a);
        u.y = *reinterpret_cast<uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(p) = u;
    }
};
template <> struct RowIO<float, 4> {
    static __device__ __forceinline__ void load(const float *p, float *f) {
        float4 v = *reinterpret_cast<const float4 *>(p);
        f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    }
    static __device__ __forceinline__ void store(float *p, const float *f) {
        *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
    }
};

constexpr int ROW_THREADS = 256;  // 8 warps, one row each

// Row (b, t, h) of flat warp index idx over all rows ([B, Tq, H], h fastest) or,
// with a q_tiles list, over B x segments x 128 x H (rows past a segment's count,
// and segments out of range, give false).
__device__ __forceinline__ bool row_of(const Problem &P, int64_t idx, int &b, int &t, int &h) {
    h = (int)(idx % P.H);
    if (!P.q_tiles) {
        if (idx >= (int64_t)P.B * P.Tq * P.H) return false;
        t = (int)((idx / P.H) % P.Tq);
        b = (int)(idx / ((int64_t)P.H * P.Tq));
        return true;
    }
    const int r = (int)((idx / P.H) % 128);
    const int64_t bs = idx / ((int64_t)P.H * 128);
    if (bs >= (int64_t)P.B * P.num_q_tiles) return false;
    const int seg = (int)(bs % P.num_q_tiles);
    b = (int)(bs / P.num_q_tiles);
    int t0, n;
    if (!q_segment(P.q_tiles, P.q_tile_rows, seg, P.Tq, t0, n) || r >= n) return false;
    t = t0 + r;
    return true;
}

// Warps (rows) a row kernel covers: every row, or 128 per listed segment.
__host__ __device__ inline int64_t row_slots(const Problem &P) {
    return P.q_tiles ? (int64_t)P.B * P.num_q_tiles * 128 * P.H : (int64_t)P.B * P.Tq * P.H;
}

// Checks a q_tiles list for the backward: every entry in range (q_segment) and
// the segments sorted by start and disjoint.  Raises EAGLE_ATTN_DEV_BAD_TILE.
__global__ void check_segments_kernel(Problem P) {
    for (int i = threadIdx.x; i < P.num_q_tiles; i += blockDim.x) {
        int t0, n, t1, n1;
        if (!q_segment(P.q_tiles, P.q_tile_rows, i, P.Tq, t0, n)) {
            raise_status(EAGLE_ATTN_DEV_BAD_TILE);
        } else if (i + 1 < P.num_q_tiles && q_segment(P.q_tiles, P.q_tile_rows, i + 1, P.Tq, t1, n1) &&
                   t1 < t0 + n) {
            raise_status(EAGLE_ATTN_DEV_BAD_TILE);
        }
    }
}

// Fold diagonal blocks 1..NB-1 into the fp32 running state (NeMo AutoModel
// "eagle.ring_attention", _merge_diag: a one-key block has lse = its logit
// (Q_t . K_i_t) * scale and out = V_i_t).
template <typename T, int E>
__global__ void __launch_bounds__(ROW_THREADS) merge_diag_kernel(Problem P, const T *__restrict__ q,
                                                                const T *__restrict__ k,
                                                                const T *__restrict__ v,
                                                                float *__restrict__ out,
                                                                float *__restrict__ lse) {
    int64_t row = (int64_t)blockIdx.x * (ROW_THREADS / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= (int64_t)P.B * P.Tq * P.H) return;
    const int h = (int)(row % P.H);
    const int t = (int)((row / P.H) % P.Tq);
    const int b = (int)(row / ((int64_t)P.H * P.Tq));
    const int64_t qo = b * P.q_sb + t * P.q_st + (int64_t)h * P.D + lane * E;
    float qf[E], o[E];
    RowIO<T, E>::load(q + qo, qf);
    RowIO<float, E>::load(out + qo, o);
    const int64_t li = ((int64_t)b * P.H + h) * P.Tq + t;
    float m = lse[li];  // running (out, lse) as a max-free pair: weight 1 at m
    float l = 1.f;
    if (m == -INFINITY) { l = 0.f; }
    for (int i = 1; i < P.NB; ++i) {
        const int64_t ko = b * P.kv_sb + i * P.kv_sblk + t * P.kv_st + (int64_t)h * P.D + lane * E;
        float kf[E], vf[E];
        RowIO<T, E>::load(k + ko, kf);
        RowIO<T, E>::load(v + ko, vf);
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) part = fmaf(qf[e], kf[e], part);
        float z = warp_sum(part) * P.scale;
        float mn = fmaxf(m, z);
        float alpha = (m == -INFINITY) ? 0.f : expf(m - mn), p = expf(z - mn);
        l = l * alpha + p;
        m = mn;
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = fmaf(o[e], alpha, p * vf[e]);
    }
    float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] *= inv;
    RowIO<float, E>::store(out + qo, o);
    if (lane == 0) lse[li] = l > 0.f ? m + logf(l) : -INFINITY;
}

// One element per thread, for buffers that are not 16-byte aligned.
template <typename TO>
__global__ void finalize_scalar_kernel(const float *__restrict__ src, TO *__restrict__ dst,
                                       size_t n) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) dst[i] = from_f32<TO>(src[i]);
}

template <typename TO>
__global__ void finalize_kernel(const float *__restrict__ src, TO *__restrict__ dst, size_t n) {
    size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (i + 4 <= n) {
        float4 v = __ldcs(reinterpret_cast<const float4 *>(src + i));
        float f[4] = {v.x, v.y, v.z, v.w};
        RowIO<TO, 4>::store(dst + i, f);
    } else {
        for (; i < n; ++i) dst[i] = from_f32<TO>(src[i]);
    }
}

// D_t = dO_t . O_t (O = the merged output in `TO`), and dq_acc row <- 0
// unless dq_acc is null.
template <typename T, typename TO, int E>
__global__ void __launch_bounds__(ROW_THREADS) bwd_prep_kernel(Problem P, const T *__restrict__ dout,
                                                              const TO *__restrict__ out,
                                                              float *__restrict__ Dws,
                                                              float *__restrict__ dq_acc) {
    int64_t row = (int64_t)blockIdx.x * (ROW_THREADS / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= (int64_t)P.B * P.Tq * P.H) return;
    const int h = (int)(row % P.H);
    const int t = (int)((row / P.H) % P.Tq);
    const int b = (int)(row / ((int64_t)P.H * P.Tq));
    const int64_t qo = b * P.q_sb + t * P.q_st + (int64_t)h * P.D + lane * E;
    float g[E], o[E];
    RowIO<T, E>::load(dout + qo, g);
    RowIO<TO, E>::load(out + qo, o);
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) part = fmaf(g[e], o[e], part);
    float Dt = warp_sum(part);
    if (lane == 0) Dws[((int64_t)b * P.H + h) * P.Tq + t] = Dt;
    if (dq_acc) {  // the CUDA-core backward accumulates dQ here
        float z[E];
#pragma unroll
        for (int e = 0; e < E; ++e) z[e] = 0.f;
        RowIO<float, E>::store(dq_acc + row * P.D + lane * E, z);
    }
}

// Diagonal blocks in closed form, then dq = scale * (dq_acc + sum_i dz_i k_i):
//   p_i = exp(scale q.k_i - lse_t), dz_i = p_i (dO.v_i - D_t),
//   dk_i = scale dz_i q_t, dv_i = p_i dO_t.
// (NeMo AutoModel "eagle.ring_attention", _CachedRingAttention: "the diagonal
// grads are added in closed form".)
template <typename T, int E>
__global__ void __launch_bounds__(ROW_THREADS) bwd_diag_kernel(
    Problem P, const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
    const T *__restrict__ dout, const float *__restrict__ lse, const float *__restrict__ Dws,
    const float *__restrict__ dq_acc, T *__restrict__ dq, T *__restrict__ dk, T *__restrict__ dv) {
    int64_t row = (int64_t)blockIdx.x * (ROW_THREADS / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= (int64_t)P.B * P.Tq * P.H) return;
    const int h = (int)(row % P.H);
    const int t = (int)((row / P.H) % P.Tq);
    const int b = (int)(row / ((int64_t)P.H * P.Tq));
    const int64_t qo = b * P.q_sb + t * P.q_st + (int64_t)h * P.D + lane * E;
    const int64_t li = ((int64_t)b * P.H + h) * P.Tq + t;
    float qf[E], g[E], acc[E];
    RowIO<T, E>::load(q + qo, qf);
    RowIO<T, E>::load(dout + qo, g);
    RowIO<float, E>::load(dq_acc + row * P.D + lane * E, acc);
    const float L = lse[li], Dt = Dws[li];
    for (int i = 1; i < P.NB; ++i) {
        const int64_t ko = b * P.kv_sb + i * P.kv_sblk + t * P.kv_st + (int64_t)h * P.D + lane * E;
        float kf[E], vf[E];
        RowIO<T, E>::load(k + ko, kf);
        RowIO<T, E>::load(v + ko, vf);
        float a = 0.f, c = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            a = fmaf(qf[e], kf[e], a);
            c = fmaf(g[e], vf[e], c);
        }
        float z = warp_sum(a) * P.scale, dp = warp_sum(c);
        float p = (L == -INFINITY) ? 0.f : expf(z - L);
        float dz = p * (dp - Dt);
        float gk[E], gv[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            acc[e] = fmaf(dz, kf[e], acc[e]);
            gk[e] = P.scale * dz * qf[e];
            gv[e] = p * g[e];
        }
        RowIO<T, E>::store(dk + ko, gk);
        RowIO<T, E>::store(dv + ko, gv);
    }
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] *= P.scale;
    RowIO<T, E>::store(dq + qo, acc);
}

// One pass over the rows before the tensor-core backward: D_t = dO_t . O_t,
// the diagonal blocks in closed form (p_i = exp(scale q.k_i - lse_t),
// dz_i = p_i (dO.v_i - D_t), dk_i = scale dz_i q_t, dv_i = p_i dO_t) and the
// unscaled sum_i dz_i k_i that the dQ kernel starts its accumulator from
// (dq_diag, fp32 [B, H, Tq, D]).  (NeMo AutoModel "eagle.ring_attention",
// _CachedRingAttention: "the diagonal grads are added in closed form".)
// dk / dv of the diagonal blocks in GT: T (written), or fp32 with P.grad_accum
// (added to what the buffers hold).  With zero_dq, dq_diag is written (zeros)
// also when there are no diagonal blocks.  With a q_tiles list, the listed rows
// only.
// Eight blocks (64 warps) per SM when the gradients are bf16: the row pass is
// bound by the loads each SM keeps in flight, and 32 registers leave room for
// all of them (the fp32-gradient form would spill there).
template <typename T, typename TO, typename GT, int E>
__global__ void __launch_bounds__(ROW_THREADS, sizeof(GT) == 2 ? 8 : 1) bwd_rows_kernel(
    Problem P, const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
    const T *__restrict__ dout, const TO *__restrict__ out, const float *__restrict__ lse,
    float *__restrict__ Dws, float *__restrict__ dq_diag, GT *__restrict__ dk,
    GT *__restrict__ dv, int zero_dq) {
    const int64_t idx = (int64_t)blockIdx.x * (ROW_THREADS / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    int b, t, h;
    if (!row_of(P, idx, b, t, h)) return;
    const int64_t qo = b * P.q_sb + t * P.q_st + (int64_t)h * P.D + lane * E;
    const int64_t li = ((int64_t)b * P.H + h) * P.Tq + t;
    float qf[E], g[E], o[E], acc[E];
    RowIO<T, E>::load(dout + qo, g);
    RowIO<TO, E>::load(out + qo, o);
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) part = fmaf(g[e], o[e], part);
    const float Dt = warp_sum(part);
    if (lane == 0) Dws[li] = Dt;
    if (P.NB < 2) {
        if (zero_dq) {  // the accumulator the five-product backward adds into
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = 0.f;
            RowIO<float, E>::store(dq_diag + li * P.D + lane * E, acc);
        }
        return;
    }
    RowIO<T, E>::load(q + qo, qf);
    const float L = lse[li];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    for (int i = 1; i < P.NB; ++i) {
        const int64_t ko = b * P.kv_sb + i * P.kv_sblk + t * P.kv_st + (int64_t)h * P.D + lane * E;
        float kf[E], vf[E];
        RowIO<T, E>::load(k + ko, kf);
        RowIO<T, E>::load(v + ko, vf);
        float a = 0.f, c = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            a = fmaf(qf[e], kf[e], a);
            c = fmaf(g[e], vf[e], c);
        }
        const float z = warp_sum(a) * P.scale, dp = warp_sum(c);
        const float p = (L == -INFINITY) ? 0.f : expf(z - L);
        const float dz = p * (dp - Dt);
        float gk[E], gv[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            acc[e] = fmaf(dz, kf[e], acc[e]);
            gk[e] = P.scale * dz * qf[e];
            gv[e] = p * g[e];
        }
        if (P.grad_accum) {
            float ok_[E], ov[E];
            RowIO<GT, E>::load(dk + ko, ok_);
            RowIO<GT, E>::load(dv + ko, ov);
#pragma unroll
            for (int e = 0; e < E; ++e) {
                gk[e] += ok_[e];
                gv[e] += ov[e];
            }
        }
        RowIO<GT, E>::store(dk + ko, gk);
        RowIO<GT, E>::store(dv + ko, gv);
    }
    RowIO<float, E>::store(dq_diag + li * P.D + lane * E, acc);
}

// dq_t = scale * dq_acc_t, the fp32 accumulator ([B, H, Tq, D]) that the
// five-product backward added its dS K products to (it started from the
// diagonal blocks' sum_i dz_i k_i): written in GT, or added to the fp32 dq
// with P.grad_accum.  With a q_tiles list, the listed rows only.
template <typename GT, int E>
__global__ void __launch_bounds__(ROW_THREADS) dq_finalize_kernel(Problem P,
                                                                 const float *__restrict__ dq_acc,
                                                                 GT *__restrict__ dq) {
    const int64_t idx = (int64_t)blockIdx.x * (ROW_THREADS / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    int b, t, h;
    if (!P.q_tiles) {
        // rows in the accumulator's order (b, h, t): consecutive warps read
        // consecutive accumulator rows, the larger of the two streams
        if (idx >= (int64_t)P.B * P.H * P.Tq) return;
        t = (int)(idx % P.Tq);
        h = (int)((idx / P.Tq) % P.H);
        b = (int)(idx / ((int64_t)P.H * P.Tq));
    } else if (!row_of(P, idx, b, t, h)) {
        return;
    }
    const int64_t qo = b * P.q_sb + t * P.q_st + (int64_t)h * P.D + lane * E;
    const int64_t li = ((int64_t)b * P.H + h) * P.Tq + t;
    float a[E];
    RowIO<float, E>::load(dq_acc + li * P.D + lane * E, a);
#pragma unroll
    for (int e = 0; e < E; ++e) a[e] *= P.scale;
    if (P.grad_accum) {
        float o[E];
        RowIO<GT, E>::load(dq + qo, o);
#pragma unroll
        for (int e = 0; e < E; ++e) a[e] += o[e];
    }
    RowIO<GT, E>::store(dq + qo, a);
}

// One warp waits, with the pipelines' bounded wait, on an mbarrier nothing
// arrives at: the wait gives up after limit_ns and raises DEV_TIMEOUT.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        abort = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) sm100::mbar_wait(&bar, 0, (volatile int *)&abort, limit_ns);
    __syncthreads();
}

// Checks cu_seqlens once per call: cu[0] == 0, non-decreasing, every length
// <= max_seqlen, and every query / key position inside [0, cu[num_docs]).
__global__ void check_cu_kernel(const int32_t *__restrict__ cu, int nd, int max_seqlen,
                                int64_t qlo, int64_t qhi, int64_t klo, int64_t khi) {
    for (int d = threadIdx.x; d <= nd; d += blockDim.x) {
        int c = cu[d];
        if (d == 0 && c != 0) raise_status(EAGLE_ATTN_DEV_BAD_CU_SEQLENS);
        if (d > 0) {
            int len = c - cu[d - 1];
            if (len < 0) raise_status(EAGLE_ATTN_DEV_BAD_CU_SEQLENS);
            else if (max_seqlen > 0 && len > max_seqlen) raise_status(EAGLE_ATTN_DEV_DOC_TOO_LONG);
        }
        if (d == nd) {
            if (qlo < 0 || klo < 0 || qhi > c || khi > c) raise_status(EAGLE_ATTN_DEV_POS_OUTSIDE);
        }
    }
}

}  // namespace eagle
