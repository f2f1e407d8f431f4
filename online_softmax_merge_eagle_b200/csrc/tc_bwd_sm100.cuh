// tc_bwd_sm100.cuh -- tensor-core backward of the joint softmax for sm_100a.
//
// The block-0 backward runs against the MERGED lse (NeMo AutoModel
// "eagle.ulysses_attention", _block0_backward; "eagle.zigzag_ring_attention",
// zigzag_ring_flash_attn_varlen_backward): with P_ts = exp(scale q_t.k_s - lse_t),
// dP_ts = dO_t.v_s and dS_ts = P_ts (dP_ts - D_t), D_t = dO_t.O_t,
//   dV_s = sum_t P_ts dO_t,  dK_s = scale sum_t dS_ts q_t,  dQ_t = scale sum_s dS_ts k_s.
// Two deterministic kernels (no atomics), both stepping 128 x 128 tiles:
//   dkdv_kernel  one CTA per 128 keys; steps over 128-row query slices:
//                S^T = K Q^T and dP^T = V dO^T into TMEM, P^T and dS^T as
//                bf16 written back over them, then dV += P^T dO and
//                dK += dS^T Q accumulate in TMEM (A operands read from TMEM).
//                MMA order dV_i, S^T_{i+1}, dK_i, dP^T_{i+1}: two MMAs are
//                queued while the element-wise warps work on each half step.
//   dq_kernel    one CTA per 128 query rows; steps over 128-key slices:
//                S = Q K^T (two TMEM buffers) and dP = dO V^T into TMEM, dS as
//                bf16 over S, dQ += dS K in TMEM (A from TMEM), which starts
//                from the diagonal blocks' sum_i dz_i k_i (computed in closed
//                form by bwd_rows_kernel; NeMo AutoModel "eagle.ring_attention",
//                _CachedRingAttention).
// Warp roles in both: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer
// (one thread), warps 2-5 the element-wise work (one TMEM lane per thread).
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace eagle {
namespace tcbwd {

using namespace sm100;

constexpr int EW = 4;                     // element-wise warpgroups
constexpr int EW_THREADS = 128 * EW;      // one TMEM lane x column slice per thread
constexpr int THREADS = 64 + EW_THREADS;  // + producer warp + MMA warp
constexpr int MAX_DIAG = 64;

// Barrier of the element-wise warps (named barrier 1) that also ANDs `v` over
// them, so that every warp takes the same exit decision.
__device__ __forceinline__ bool group_all(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(EW_THREADS)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > 100000000ull) return;
}

__device__ __forceinline__ void bf16x8_to_f32(uint4 u, float *f) {
    const uint32_t *p = &u.x;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(p[i] << 16);
        f[2 * i + 1] = __uint_as_float(p[i] & 0xffff0000u);
    }
}

// Adds 16 fp32 values * s to 16 fp32 values in global memory (64 bytes).
__device__ __forceinline__ void add_row16_f32(float *dst, const float *v, float s) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float4 u = reinterpret_cast<const float4 *>(dst)[c];
        u.x = fmaf(v[c * 4 + 0], s, u.x);
        u.y = fmaf(v[c * 4 + 1], s, u.y);
        u.z = fmaf(v[c * 4 + 2], s, u.z);
        u.w = fmaf(v[c * 4 + 3], s, u.w);
        reinterpret_cast<float4 *>(dst)[c] = u;
    }
}

// Gradient row chunk out: bf16 written, or (P.grad_accum) fp32 added.
__device__ __forceinline__ void grad_out16(const Problem &P, void *base, int64_t off,
                                           const float *v, float s);

// Writes 16 fp32 values * s as bf16 (32 bytes) to global memory.
__device__ __forceinline__ void store_row16_bf16(__nv_bfloat16 *dst, const float *v, float s) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        uint4 u;
        u.x = pack_bf16(v[c * 8 + 0] * s, v[c * 8 + 1] * s);
        u.y = pack_bf16(v[c * 8 + 2] * s, v[c * 8 + 3] * s);
        u.z = pack_bf16(v[c * 8 + 4] * s, v[c * 8 + 5] * s);
        u.w = pack_bf16(v[c * 8 + 6] * s, v[c * 8 + 7] * s);
        reinterpret_cast<uint4 *>(dst)[c] = u;
    }
}

__device__ __forceinline__ void grad_out16(const Problem &P, void *base, int64_t off,
                                           const float *v, float s) {
    if (P.grad_accum)
        add_row16_f32(reinterpret_cast<float *>(base) + off, v, s);
    else
        store_row16_bf16(reinterpret_cast<__nv_bfloat16 *>(base) + off, v, s);
}

// Writes 32 fp32 values * s as bf16 (64 bytes) to global memory.
__device__ __forceinline__ void store_row32_bf16(__nv_bfloat16 *dst, const float *v, float s) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 u;
        u.x = pack_bf16(v[c * 8 + 0] * s, v[c * 8 + 1] * s);
        u.y = pack_bf16(v[c * 8 + 2] * s, v[c * 8 + 3] * s);
        u.z = pack_bf16(v[c * 8 + 4] * s, v[c * 8 + 5] * s);
        u.w = pack_bf16(v[c * 8 + 6] * s, v[c * 8 + 7] * s);
        reinterpret_cast<uint4 *>(dst)[c] = u;
    }
}

// ============================================================== dK / dV ===
namespace kv {

constexpr int BN = 128;  // keys per CTA (TMEM lanes)
constexpr int BM = 128;  // query rows per step
constexpr int QS = 2;    // Q / dO ring depth

template <int D>
struct Cfg {
    static constexpr int KT = BN * D * 2;  // K or V tile bytes
    static constexpr int QT = BM * D * 2;  // Q or dO slice bytes
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + KT;
    static constexpr int OFF_Q = OFF_V + KT;
    static constexpr int OFF_DO = OFF_Q + QS * QT;
    static constexpr int OFF_ROW = OFF_DO + QS * QT;  // lse2, D, lo, hi + 2 scalars per stage
    static constexpr int ROW_BYTES = 4 * BM * 4 + 16;
    static constexpr int OFF_BAR = OFF_ROW + 2 * ROW_BYTES;
    static constexpr int NBARS = 32;  // >= the barriers laid out in the kernel
    static constexpr int SMEM = OFF_BAR + NBARS * 8 + 16 + 1024;
    static constexpr uint32_t T_DV = 0, T_DK = 128, T_ST = 256, T_DPT = 384, TMEM_COLS = 512;
};

template <int D>
__global__ void __launch_bounds__(THREADS, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const Problem P, const float *__restrict__ lse, const float *__restrict__ Dws,
                void *__restrict__ dk, void *__restrict__ dv) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = (uint64_t *)(smem + C::OFF_BAR);
    uint64_t *bar_kv = bars + 0;
    uint64_t *bar_qf = bars + 1, *bar_qe = bars + 1 + QS;  // QS each
    uint64_t *bar_stf = bars + 1 + 2 * QS;                 // S^T_i in TMEM
    uint64_t *bar_dpf = bar_stf + 1;                       // dP^T_i in TMEM
    uint64_t *bar_ptf = bar_dpf + 1;                       // P^T_i written over S^T_i
    uint64_t *bar_dsf = bar_ptf + 1;                       // dS^T_i written over dP^T_i
    uint64_t *bar_done = bar_dsf + 1;
    static_assert(C::NBARS >= 1 + 2 * QS + 5, "barrier slots");
    uint32_t *tmem_slot = (uint32_t *)(bars + C::NBARS);
    volatile int *abort = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int kt, pr;  // grid (key tiles, H, B), heaviest key tiles first
    heavy_first(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z), gridDim.x,
                gridDim.y * gridDim.z, kt, pr);
    const int ks = kt * BN, h = pr % gridDim.y, b = pr / gridDim.y;
    int tbeg, tend;
    keys_row_range(P.mask, ks, min(ks + BN, P.Tk) - 1, tbeg, tend);
    const int nsteps = tend >= tbeg ? (tend - tbeg + BM) / BM : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NBARS; ++i) mbar_init(&bars[i], 1);
        mbar_init(bar_ptf, EW_THREADS);
        mbar_init(bar_dsf, EW_THREADS);
        *abort = status_bad() ? 1 : 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool skip = *abort != 0;

    if (warp == 0) {
        // ------------------------------------------------------ producer --
        if (lane == 0 && !skip) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_do);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_expect_tx(bar_kv, 2 * C::KT);
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
                tma_load_5d(smem + C::OFF_K + cb * BN * 128, &tm_k, bar_kv, cb * 64, h, ks, 0, b);
                tma_load_5d(smem + C::OFF_V + cb * BN * 128, &tm_v, bar_kv, cb * 64, h, ks, 0, b);
            }
            int issued = 0;
            for (int i = 0; i < nsteps; ++i) {
                const int st = i % QS;
                const int t0 = tbeg + i * BM;
                if (!mbar_wait(bar_qe + st, ((i / QS) & 1) ^ 1, abort)) break;
                mbar_expect_tx(bar_qf + st, 2 * C::QT);
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb) {
                    tma_load_4d(smem + C::OFF_Q + st * C::QT + cb * BM * 128, &tm_q, bar_qf + st,
                                cb * 64, h, t0, b);
                    tma_load_4d(smem + C::OFF_DO + st * C::QT + cb * BM * 128, &tm_do, bar_qf + st,
                                cb * 64, h, t0, b);
                }
                issued = i + 1;
            }
            if (*abort) {
                drain_wait(bar_kv, 0);
                for (int i = (issued > QS ? issued - QS : 0); i < issued; ++i)
                    drain_wait(bar_qf + i % QS, (i / QS) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA ---
        if (lane == 0 && !skip) {
            const uint32_t id_st = idesc_bf16(BN, BM, false);  // M=128 keys, N=128 rows
            const uint32_t id_acc = idesc_bf16(BN, D, true);   // M=128 keys, N=D, B MN-major
            const uint32_t k_s = smem_u32(smem + C::OFF_K), v_s = smem_u32(smem + C::OFF_V);
            const uint32_t q_s = smem_u32(smem + C::OFF_Q), do_s = smem_u32(smem + C::OFF_DO);
            bool ok = mbar_wait(bar_kv, 0, abort);
            // S^T_i = K Q_i^T (waits for the slice), dP^T_i = V dO_i^T
            auto issue_st = [&](int i) -> bool {
                const int st = i % QS;
                if (!mbar_wait(bar_qf + st, (i / QS) & 1, abort)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
                    umma_ss(tmem + C::T_ST, sdesc_sw128(k_s + off, 16, 1024),
                            sdesc_sw128(q_s + st * C::QT + off, 16, 1024), id_st, kk > 0);
                }
                umma_commit(bar_stf);
                return true;
            };
            auto issue_dpt = [&](int i) {
                const int st = i % QS;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
                    umma_ss(tmem + C::T_DPT, sdesc_sw128(v_s + off, 16, 1024),
                            sdesc_sw128(do_s + st * C::QT + off, 16, 1024), id_st, kk > 0);
                }
                umma_commit(bar_dpf);
            };
            // P^T_i / dS^T_i: rows [32g, 32g + 32) packed into columns [32g, 32g + 16)
            // of the S^T / dP^T buffer they replaced
            auto issue_dv = [&](int i) -> bool {
                const int st = i % QS;
                if (!mbar_wait(bar_ptf, i & 1, abort)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < BM / 16; ++kk)
                    umma_ts(tmem + C::T_DV, tmem + C::T_ST + (kk >> 1) * 32 + (kk & 1) * 8,
                            sdesc_sw128(do_s + st * C::QT + kk * 2048, BM * 128, 1024), id_acc,
                            (i > 0 || kk > 0) ? 1u : 0u);
                return true;
            };
            auto issue_dk = [&](int i) -> bool {
                const int st = i % QS;
                if (!mbar_wait(bar_dsf, i & 1, abort)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < BM / 16; ++kk)
                    umma_ts(tmem + C::T_DK, tmem + C::T_DPT + (kk >> 1) * 32 + (kk & 1) * 8,
                            sdesc_sw128(q_s + st * C::QT + kk * 2048, BM * 128, 1024), id_acc,
                            (i > 0 || kk > 0) ? 1u : 0u);
                umma_commit(bar_qe + st);
                return true;
            };
            if (ok && nsteps > 0) {
                ok = issue_st(0);
                if (ok) issue_dpt(0);
                for (int i = 0; ok && i < nsteps; ++i) {
                    // the next S^T / dP^T overwrite P^T_i / dS^T_i: issued after the
                    // MMA that reads them (the tensor pipe runs them in order)
                    ok = issue_dv(i);
                    if (ok && i + 1 < nsteps) ok = issue_st(i + 1);
                    if (ok) ok = issue_dk(i);
                    if (ok && i + 1 < nsteps) issue_dpt(i + 1);
                }
            }
            umma_commit(bar_done);
            drain_wait(bar_done, 0);
        }
    } else {
        // -------------------------------------------- element-wise (key) ---
        // thread = (key = TMEM lane, quarter of the 128 rows of a step)
        const int quad = warp & 3;
        const int eg = (warp - 2) >> 2;   // which 32 rows of the step
        const int sl = quad * 32 + lane;  // key within the tile
        const int s = ks + sl;            // local key index
        const int tid = threadIdx.x - 64; // 0 .. EW_THREADS-1
        const float sl2 = P.scale * 1.4426950408889634f;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        constexpr int HC = BM / EW;       // 32 rows per thread and step
        // Row data of a step (lse in the exp2 domain, D_t, the row's key
        // interval, and the step's fully-visible key range), gathered by
        // threads 0..127 a step ahead.  The loads are only issued here; their
        // values are first used when the next step writes them to shared memory.
        struct RowData {
            float L, dd;
            int lo, hi, flo, fhi;
        };
        auto gather = [&](int i) -> RowData {
            RowData d{-INFINITY, 0.f, 1, 0, 1, 0};
            const int t0 = tbeg + i * BM;
            const int t = t0 + tid;
            if (tid < BM && i < nsteps && t <= tend && t < P.Tq) {
                if (row_interval(P.mask, t, d.lo, d.hi) != 0) { d.lo = 1; d.hi = 0; }
                d.L = __ldg(lse + ((int64_t)b * P.H + h) * P.Tq + t);
                d.dd = __ldg(Dws + ((int64_t)b * P.H + h) * P.Tq + t);
            }
            if (tid == 0 && i < nsteps) {
                // every row of the step valid: the interval ends are monotone, so the
                // step is fully visible to keys in [lo(last row), hi(first row)]
                const int tl_ = t0 + BM - 1;
                int lo1 = 1, hi1 = 0, lo0 = 1, hi0 = 0;
                if (tl_ <= tend && tl_ < P.Tq && row_interval(P.mask, tl_, lo1, hi1) == 0 &&
                    row_interval(P.mask, t0, lo0, hi0) == 0) {
                    d.flo = lo1;
                    d.fhi = hi0;
                }
            }
            return d;
        };
        RowData next = gather(0);
        bool ok = !skip;
        for (int i = 0; i < nsteps; ++i) {
            const int bi = i & 1;
            float *r_lse = reinterpret_cast<float *>(smem + C::OFF_ROW + bi * C::ROW_BYTES);
            float *r_d = r_lse + BM;
            int *r_lo = reinterpret_cast<int *>(r_d + BM);
            int *r_hi = r_lo + BM;
            int *r_full = r_hi + BM;  // [0] = largest lo, [1] = smallest hi of the step
            if (ok && tid < BM) {
                r_lse[tid] = (next.L == -INFINITY) ? INFINITY : next.L * 1.4426950408889634f;
                r_d[tid] = next.dd;
                r_lo[tid] = next.lo;
                r_hi[tid] = next.hi;
                if (tid == 0) {
                    r_full[0] = next.flo;
                    r_full[1] = next.fhi;
                }
            }
            ok = group_all(ok);  // row data written; all element-wise warps agree to go on
            if (!ok) break;
            next = gather(i + 1);  // after the barrier, which would wait for these loads
            ok = __all_sync(0xffffffffu, mbar_wait(bar_stf, i & 1, abort));
            if (!ok) continue;
            tc_fence_after();
            uint32_t v[HC];
            tmem_ldn<HC>(tl + C::T_ST + eg * HC, v);
            tmem_ld_wait();
            const bool full = r_full[0] <= s && s <= r_full[1];
            const float *cl = r_lse + eg * HC;
            float p[HC];
            if (full) {
#pragma unroll
                for (int r = 0; r < HC; ++r) p[r] = ex2(fmaf(__uint_as_float(v[r]), sl2, -cl[r]));
            } else {
                const int *clo = r_lo + eg * HC, *chi = r_hi + eg * HC;
#pragma unroll
                for (int r = 0; r < HC; ++r) {
                    const bool vis = (clo[r] <= s) && (s <= chi[r]);
                    p[r] = vis ? ex2(fmaf(__uint_as_float(v[r]), sl2, -cl[r])) : 0.f;
                }
            }
            // P^T (this key, these rows) as bf16 pairs over this thread's S^T columns
            {
                uint32_t pk[HC / 2];
#pragma unroll
                for (int c = 0; c < HC / 2; ++c) pk[c] = pack_bf16(p[2 * c], p[2 * c + 1]);
                tmem_stn<HC / 2>(tl + C::T_ST + eg * HC, pk);
                tmem_st_wait();
            }
            tc_fence_before();
            mbar_arrive(bar_ptf);
            ok = __all_sync(0xffffffffu, mbar_wait(bar_dpf, i & 1, abort));
            if (!ok) continue;
            tc_fence_after();
            tmem_ldn<HC>(tl + C::T_DPT + eg * HC, v);
            tmem_ld_wait();
            const float *cd = r_d + eg * HC;
#pragma unroll
            for (int r = 0; r < HC; ++r) p[r] = p[r] * (__uint_as_float(v[r]) - cd[r]);
            {
                uint32_t pk[HC / 2];
#pragma unroll
                for (int c = 0; c < HC / 2; ++c) pk[c] = pack_bf16(p[2 * c], p[2 * c + 1]);
                tmem_stn<HC / 2>(tl + C::T_DPT + eg * HC, pk);
                tmem_st_wait();
            }
            tc_fence_before();
            mbar_arrive(bar_dsf);
        }
        // ------------------------------------------------------ epilogue ---
        // each warpgroup writes a quarter of the D columns of its keys' dV and dK
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, abort));
        tc_fence_after();
        constexpr int NCH = D / 16 / EW;  // 16-column chunks per warpgroup
#pragma unroll 1
        for (int q = 0; q < 2 * NCH; ++q) {  // dV chunks, then dK chunks
            const int c = eg * NCH + (q % NCH);
            const bool is_k = q >= NCH;
            uint32_t a[16];
            if (ok && nsteps > 0) {
                tmem_ldn<16>(tl + (is_k ? C::T_DK : C::T_DV) + c * 16, a);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) a[e] = 0u;
            }
            if (ok && s < P.Tk) {
                const int64_t off = b * P.kv_sb + (int64_t)s * P.kv_st + (int64_t)h * D + c * 16;
                grad_out16(P, is_k ? dk : dv, off, reinterpret_cast<const float *>(a),
                           is_k ? P.scale : 1.f);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace kv

// ================================================================== dQ ===
namespace qk {

constexpr int BM = 128;  // query rows per CTA (TMEM lanes)
constexpr int BN = 128;  // keys per step
constexpr int KS = 3;    // K ring depth: a K slice lives from S_j to dQ_j
constexpr int VS = 2;    // V ring depth: a V slice lives from dP_j only

template <int D>
struct Cfg {
    static constexpr int QT = BM * D * 2;
    static constexpr int KT = BN * D * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_DO = QT;
    static constexpr int OFF_K = 2 * QT;
    static constexpr int OFF_V = OFF_K + KS * KT;
    static constexpr int OFF_BAR = OFF_V + VS * KT;
    static constexpr int NBARS = 32;  // >= the barriers laid out in the kernel
    static constexpr int SMEM = OFF_BAR + NBARS * 8 + 16 + 1024;
    static constexpr uint32_t T_S = 0, T_DP = 256, T_DQ = 384, TMEM_COLS = 512;
};

template <int D>
__global__ void __launch_bounds__(THREADS, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const Problem P, const float *__restrict__ lse, const float *__restrict__ Dws,
              const float *__restrict__ dq_diag, void *__restrict__ dq) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = (uint64_t *)(smem + C::OFF_BAR);
    uint64_t *bar_q = bars + 0;
    uint64_t *bar_kf = bars + 1, *bar_ke = bar_kf + KS;   // KS each
    uint64_t *bar_vf = bar_ke + KS, *bar_ve = bar_vf + VS; // VS each
    uint64_t *bar_sf = bar_ve + VS;                        // 2: S_j in TMEM buffer j & 1
    uint64_t *bar_dpf = bar_sf + 2, *bar_dpe = bar_dpf + 1;  // dP_j in / read from TMEM
    uint64_t *bar_dsf = bar_dpe + 1;                       // 2: dS_j written over S_j
    uint64_t *bar_done = bar_dsf + 2;
    static_assert(C::NBARS >= 1 + 2 * KS + 2 * VS + 7, "barrier slots");
    uint32_t *tmem_slot = (uint32_t *)(bars + C::NBARS);
    volatile int *abort = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_qtiles = (P.Tq + BM - 1) / BM;
    int qt, pr;  // grid (query tiles, H, B), heaviest (last) query tiles first
    heavy_first(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z), gridDim.x,
                gridDim.y * gridDim.z, qt, pr);
    const int t0 = (n_qtiles - 1 - qt) * BM;
    const int h = pr % gridDim.y, b = pr / gridDim.y;
    int kbeg, kend;
    rows_key_range(P.mask, t0, min(t0 + BM, P.Tq) - 1, kbeg, kend);
    const int nsteps = kend >= kbeg ? (kend - kbeg + BN) / BN : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NBARS; ++i) mbar_init(&bars[i], 1);
        mbar_init(bar_dpe, EW_THREADS);
        mbar_init(bar_dsf + 0, EW_THREADS);
        mbar_init(bar_dsf + 1, EW_THREADS);
        *abort = status_bad() ? 1 : 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool skip = *abort != 0;

    if (warp == 0) {
        // ------------------------------------------------------ producer --
        if (lane == 0 && !skip) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_do);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_expect_tx(bar_q, 2 * C::QT);
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
                tma_load_4d(smem + C::OFF_Q + cb * BM * 128, &tm_q, bar_q, cb * 64, h, t0, b);
                tma_load_4d(smem + C::OFF_DO + cb * BM * 128, &tm_do, bar_q, cb * 64, h, t0, b);
            }
            int kiss = 0, viss = 0;  // slices issued
            for (int j = 0; j < nsteps; ++j) {
                const int k0 = kbeg + j * BN;
                const int sk = j % KS, sv = j % VS;
                if (!mbar_wait(bar_ke + sk, ((j / KS) & 1) ^ 1, abort)) break;
                mbar_expect_tx(bar_kf + sk, C::KT);
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_5d(smem + C::OFF_K + sk * C::KT + cb * BN * 128, &tm_k, bar_kf + sk,
                                cb * 64, h, k0, 0, b);
                kiss = j + 1;
                if (!mbar_wait(bar_ve + sv, ((j / VS) & 1) ^ 1, abort)) break;
                mbar_expect_tx(bar_vf + sv, C::KT);
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_5d(smem + C::OFF_V + sv * C::KT + cb * BN * 128, &tm_v, bar_vf + sv,
                                cb * 64, h, k0, 0, b);
                viss = j + 1;
            }
            if (*abort) {
                drain_wait(bar_q, 0);
                for (int j = (kiss > KS ? kiss - KS : 0); j < kiss; ++j)
                    drain_wait(bar_kf + j % KS, (j / KS) & 1);
                for (int j = (viss > VS ? viss - VS : 0); j < viss; ++j)
                    drain_wait(bar_vf + j % VS, (j / VS) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA ---
        if (lane == 0 && !skip) {
            const uint32_t id_s = idesc_bf16(BM, BN, false);  // M=128 rows, N=128 keys
            const uint32_t id_q = idesc_bf16(BM, D, true);    // M=128 rows, N=D, B MN-major
            const uint32_t q_s = smem_u32(smem + C::OFF_Q), do_s = smem_u32(smem + C::OFF_DO);
            const uint32_t k_s = smem_u32(smem + C::OFF_K), v_s = smem_u32(smem + C::OFF_V);
            bool ok = mbar_wait(bar_q, 0, abort);
            auto issue_s = [&](int j) -> bool {
                const int sk = j % KS;
                if (!mbar_wait(bar_kf + sk, (j / KS) & 1, abort)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                    umma_ss(tmem + C::T_S + (j & 1) * BN, sdesc_sw128(q_s + off, 16, 1024),
                            sdesc_sw128(k_s + sk * C::KT + off, 16, 1024), id_s, kk > 0);
                }
                umma_commit(bar_sf + (j & 1));
                return true;
            };
            // dP_j into the single dP buffer: every element-wise thread has read dP_{j-1}
            auto issue_dp = [&](int j) -> bool {
                const int sv = j % VS;
                if (!mbar_wait(bar_vf + sv, (j / VS) & 1, abort)) return false;
                if (j > 0 && !mbar_wait(bar_dpe, (j - 1) & 1, abort)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                    umma_ss(tmem + C::T_DP, sdesc_sw128(do_s + off, 16, 1024),
                            sdesc_sw128(v_s + sv * C::KT + off, 16, 1024), id_s, kk > 0);
                }
                umma_commit(bar_dpf);
                umma_commit(bar_ve + sv);
                return true;
            };
            // dS_j: keys [32g, 32g + 32) packed into columns [32g, 32g + 16) of the
            // S_j buffer they replaced
            auto issue_dq = [&](int j) -> bool {
                const int sk = j % KS;
                if (!mbar_wait(bar_dsf + (j & 1), (j >> 1) & 1, abort)) return false;
                tc_fence_after();
                const uint32_t a = tmem + C::T_S + (j & 1) * BN;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    umma_ts(tmem + C::T_DQ, a + (kk >> 1) * 32 + (kk & 1) * 8,
                            sdesc_sw128(k_s + sk * C::KT + kk * 2048, BN * 128, 1024), id_q,
                            (j > 0 || kk > 0 || dq_diag) ? 1u : 0u);
                umma_commit(bar_ke + sk);
                return true;
            };
            if (ok && nsteps > 0) {
                ok = issue_s(0);
                if (ok) ok = issue_dp(0);
                for (int j = 0; ok && j < nsteps; ++j) {
                    // S_{j+1} goes to the other buffer; S_{j+2} (next iteration)
                    // overwrites dS_j only after dQ_j, in tensor-pipe order
                    if (j + 1 < nsteps) ok = issue_s(j + 1);
                    if (ok && j + 1 < nsteps) ok = issue_dp(j + 1);
                    if (ok) ok = issue_dq(j);
                }
            }
            umma_commit(bar_done);
            drain_wait(bar_done, 0);
        }
    } else {
        // -------------------------------------------- element-wise (row) ---
        // thread = (row = TMEM lane, quarter of the 128 keys of a step)
        const int quad = warp & 3;
        const int eg = (warp - 2) >> 2;
        const int r = quad * 32 + lane;
        const int t = t0 + r;
        const bool valid = t < P.Tq;
        constexpr int HC = BN / EW;  // 32 keys per thread and step
        int lo = 1, hi = 0;
        if (valid && row_interval(P.mask, t, lo, hi) != 0) { lo = 1; hi = 0; }
        const int64_t li = ((int64_t)b * P.H + h) * P.Tq + t;
        const float L = valid ? lse[li] : -INFINITY;
        const float l2 = (L == -INFINITY) ? INFINITY : L * 1.4426950408889634f;
        const float Dt = valid ? Dws[li] : 0.f;
        const float sl2 = P.scale * 1.4426950408889634f;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        constexpr int NCH = D / 16 / EW;  // 16-column chunks of dQ per warpgroup
        bool ok = !skip;
        if (dq_diag && ok) {
            // dQ starts from the diagonal blocks' sum_i dz_i k_i of this row; the
            // first dQ MMA waits for dsf, which this thread signals after the store
            const float4 *src = reinterpret_cast<const float4 *>(
                dq_diag + (valid ? li : 0) * (int64_t)D + eg * (D / EW));
#pragma unroll
            for (int cc = 0; cc < NCH; ++cc) {
                uint32_t a[16];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 f = valid ? __ldg(src + cc * 4 + u) : make_float4(0.f, 0.f, 0.f, 0.f);
                    a[u * 4] = __float_as_uint(f.x);
                    a[u * 4 + 1] = __float_as_uint(f.y);
                    a[u * 4 + 2] = __float_as_uint(f.z);
                    a[u * 4 + 3] = __float_as_uint(f.w);
                }
                tmem_stn<16>(tl + C::T_DQ + (eg * NCH + cc) * 16, a);
            }
            tmem_st_wait();
        }
        for (int j = 0; ok && j < nsteps; ++j) {
            const int bj = j & 1;
            const int k0 = kbeg + j * BN + eg * HC;  // first key of this thread's quarter
            ok = __all_sync(0xffffffffu, mbar_wait(bar_sf + bj, (j >> 1) & 1, abort));
            if (!ok) break;
            tc_fence_after();
            uint32_t v[HC];
            tmem_ldn<HC>(tl + C::T_S + bj * BN + eg * HC, v);
            tmem_ld_wait();
            float p[HC];
            if (lo <= k0 && k0 + HC - 1 <= hi) {
#pragma unroll
                for (int c = 0; c < HC; ++c) p[c] = ex2(fmaf(__uint_as_float(v[c]), sl2, -l2));
            } else {
#pragma unroll
                for (int c = 0; c < HC; ++c) {
                    const bool vis = k0 + c >= lo && k0 + c <= hi;
                    p[c] = vis ? ex2(fmaf(__uint_as_float(v[c]), sl2, -l2)) : 0.f;
                }
            }
            ok = __all_sync(0xffffffffu, mbar_wait(bar_dpf, j & 1, abort));
            if (!ok) break;
            tc_fence_after();
            tmem_ldn<HC>(tl + C::T_DP + eg * HC, v);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(bar_dpe);
#pragma unroll
            for (int c = 0; c < HC; ++c) p[c] = p[c] * (__uint_as_float(v[c]) - Dt);
            {
                uint32_t pk[HC / 2];
#pragma unroll
                for (int c = 0; c < HC / 2; ++c) pk[c] = pack_bf16(p[2 * c], p[2 * c + 1]);
                tmem_stn<HC / 2>(tl + C::T_S + bj * BN + eg * HC, pk);
                tmem_st_wait();
            }
            tc_fence_before();
            mbar_arrive(bar_dsf + bj);
        }
        // ---------------------------------------------------- epilogue ----
        // dq = scale (sum_s dS_ts k_s + sum_i dz_i k_i); each warpgroup writes a quarter
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, abort));
        tc_fence_after();
        const bool have = ok && (nsteps > 0 || dq_diag != nullptr);
#pragma unroll 1
        for (int cc = 0; cc < NCH; ++cc) {
            const int c = eg * NCH + cc;
            uint32_t a[16];
            if (have) {
                tmem_ldn<16>(tl + C::T_DQ + c * 16, a);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) a[e] = 0u;
            }
            if (ok && valid)
                grad_out16(P, dq, b * P.q_sb + (int64_t)t * P.q_st + (int64_t)h * D + c * 16,
                           reinterpret_cast<const float *>(a), P.scale);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace qk

// ========================================================= dK / dV / dQ ===
// The backward with five products per tile pair (the non-deterministic
// mode): one CTA per 128 keys steps over 128-row query slices as
// kv::dkdv_kernel does and, from the dS^T tile it already holds, also forms
// dQ_i = dS_i K (M = 128 rows, N = D, K = the CTA's 128 keys), which it adds
// to the fp32 dQ accumulator in global memory (the order of those fp32
// additions across CTAs varies from run to run).  dS^T goes to shared memory
// once, bf16 with the 128-byte swizzle, and serves as the K-major A operand of
// dK += dS^T Q and as the MN-major A operand of dQ_i = dS K.
// Shared memory: K, V, a ring of three Q slots and two dO slots; at D = 128
// dS^T_i is written over dO_i once dV_i has read it (at D = 64 it has a tile
// of its own).  dQ_i leaves through the slots of Q_i and dO_i, which no
// product reads once dQ_i is complete: the element-wise warps stage it there
// (fp32, in the swizzled boxes of a TMA tensor map over the accumulator), and
// the producer warp, which owns the slots, issues TMA reduce-adds (whole L2
// lines) in two bulk groups, the boxes over dO_i's slot first, and loads
// dO_{i+2} as soon as that group has read its slot and Q_{i+3} once the second
// has -- a step and two steps before they are needed, so the reductions drain
// while the next steps compute.
// TMEM: dV [0, D), dK [128, 128 + D) and two 128-column regions R0, R1 that
// carry in turn S^T_i -> P^T_i (R_{i%2}), dP^T_i (R_{(i+1)%2}) and dQ_i
// (R_{i%2}, issued after dV_i has read P^T_i).
// MMA issue order: S^T_0, dP^T_0, dV_0, then per step i: S^T_{i+1} (once the
// element-wise warps have read dP^T_i); dK_i, dQ_i (once dS^T_i is in shared
// memory); dV_{i+1} (once P^T_{i+1} is written); dP^T_{i+1} (once dQ_i has
// been read out of R_{i%2}).  The elementwise warps' order per step: P^T_i,
// then dQ_{i-1} out, then dP^T_i read and dS^T_i.
namespace kvq {

constexpr int BN = 128;  // keys per CTA (TMEM lanes of S^T, dP^T, dV, dK)
constexpr int BM = 128;  // query rows per step (TMEM lanes of dQ_i)
constexpr int QSL = 3;   // Q slots
constexpr int OSL = 2;   // dO slots
constexpr int DQ_BOX_COLS = 32;  // fp32 box of the dQ tensor map: 32 columns (128 bytes)
constexpr int DQ_BOX_ROWS = BM;  // x the 128 rows of a slice

template <int D>
struct Cfg {
    static constexpr int KT = BN * D * 2;    // K or V tile bytes
    static constexpr int QT = BM * D * 2;    // Q or dO slice bytes (one slot)
    static constexpr int DST = BN * BM * 2;  // dS^T tile bytes
    static constexpr bool DS_IN_DO = QT >= DST;  // dS^T_i over dO_i (D = 128)
    static constexpr int BOX = DQ_BOX_ROWS * DQ_BOX_COLS * 4;  // one staged dQ box
    static constexpr int NBOX = D / DQ_BOX_COLS;                // boxes per slice
    static_assert((NBOX / 2) * BOX == QT, "half the dQ boxes fill a Q (or dO) slot");
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + KT;
    static constexpr int OFF_Q = OFF_V + KT;
    static constexpr int OFF_DO = OFF_Q + QSL * QT;
    static constexpr int OFF_DS = OFF_DO + OSL * QT;  // own dS^T tile (D = 64 only)
    static constexpr int OFF_ROW = OFF_DS + (DS_IN_DO ? 0 : DST);  // two RowSlots
    static constexpr int ROW_BYTES = 2 * BM * 4 + 16;              // lse, D_t, t0, t1
    static constexpr int OFF_BAR = OFF_ROW + 2 * ROW_BYTES;
    static constexpr int NBARS = 20;  // >= the barriers laid out in the kernel
    // no realignment slack: the kernel checks that the base is 1024-byte aligned
    static constexpr int SMEM = OFF_BAR + NBARS * 8 + 16;
    static_assert(SMEM <= 232448, "shared memory");
    static constexpr uint32_t T_DV = 0, T_DK = 128, T_R0 = 256, T_R1 = 384, TMEM_COLS = 512;
    static_assert(D <= 128, "TMEM budget");
    static __device__ __forceinline__ int q_off(int i) { return OFF_Q + (i % QSL) * QT; }
    static __device__ __forceinline__ int do_off(int i) { return OFF_DO + (i % OSL) * QT; }
    static __device__ __forceinline__ int ds_off(int i) { return DS_IN_DO ? do_off(i) : OFF_DS; }
    // staged dQ box bx of slice i: the first half of the boxes over Q_i's slot,
    // the second half over dO_i's
    static __device__ __forceinline__ int box_off(int i, int bx) {
        return (bx < NBOX / 2 ? q_off(i) : do_off(i)) + (bx % (NBOX / 2)) * BOX;
    }
};

// Named barrier 2 over the element-wise warps.
__device__ __forceinline__ void ew_sync() {
    asm volatile("bar.sync 2, %0;" ::"n"(EW_THREADS) : "memory");
}

// SEG: the query slices are the segments of a q_tiles list (a separate
// instantiation, so that the whole-row path keeps its register allocation).
template <int D, bool SEG>
__global__ void __launch_bounds__(THREADS, 1)
    dkdvdq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_dq, const Problem P,
                  const float *__restrict__ lse, const float *__restrict__ Dws,
                  void *__restrict__ dk, void *__restrict__ dv) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw;
    // the swizzled tiles need a 1024-byte aligned base (CTA-uniform test; nothing
    // has been allocated or started yet)
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) raise_status(EAGLE_ATTN_DEV_SMEM_ALIGN);
        return;
    }
    uint64_t *bars = (uint64_t *)(smem + C::OFF_BAR);
    uint64_t *bar_kv = bars + 0;
    uint64_t *bar_qf = bars + 1;           // [QSL]: Q_i landed
    uint64_t *bar_of = bar_qf + QSL;       // [OSL]: dO_i landed
    uint64_t *bar_sf = bar_of + OSL;       // S^T_i in TMEM
    uint64_t *bar_dpf = bar_sf + 1;        // dP^T_i in TMEM
    uint64_t *bar_dvd = bar_dpf + 1;       // dV_i done: dO_i no longer read
    uint64_t *bar_dqf = bar_dvd + 1;       // dQ_i in TMEM (dK_i done too: dS^T free)
    uint64_t *bar_ptf = bar_dqf + 1;       // P^T_i written over S^T_i (EW_THREADS)
    uint64_t *bar_dpr = bar_ptf + 1;       // dP^T_i read out of TMEM (EW_THREADS)
    uint64_t *bar_dsf = bar_dpr + 1;       // dS^T_i in shared memory (EW_THREADS)
    uint64_t *bar_dqe = bar_dsf + 1;       // dQ_i read out of TMEM (EW_THREADS)
    uint64_t *bar_stg = bar_dqe + 1;       // dQ_i staged over Q_i and dO_i (EW_THREADS)
    uint64_t *bar_done = bar_stg + 1;
    static_assert(C::NBARS >= 1 + QSL + OSL + 11, "barrier slots");
    uint32_t *tmem_slot = (uint32_t *)(bars + C::NBARS);
    volatile int *abort = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int kt, pr;  // grid (key tiles, H, B), heaviest key tiles first
    heavy_first(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z), gridDim.x,
                gridDim.y * gridDim.z, kt, pr);
    const int ks = kt * BN, h = pr % gridDim.y, b = pr / gridDim.y;
    int tbeg, tend;
    keys_row_range(P.mask, ks, min(ks + BN, P.Tk) - 1, tbeg, tend);
    // query slices: 128 rows at a time from tbeg or, with a q_tiles list, the
    // listed segments (sorted, disjoint, <= 128 rows) that meet [tbeg, tend]
    int seg0 = 0, nsteps = tend >= tbeg ? (tend - tbeg + BM) / BM : 0;
    if (SEG) {
        auto seg_start = [&](int i) { return __ldg(P.q_tiles + i); };
        auto seg_end = [&](int i) {  // one past the last row (search only; entries checked below)
            return __ldg(P.q_tiles + i) + (P.q_tile_rows ? __ldg(P.q_tile_rows + i) : BM);
        };
        int lo = 0, hi = P.num_q_tiles;  // first segment ending after tbeg
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (seg_end(mid) > tbeg) hi = mid; else lo = mid + 1;
        }
        seg0 = lo;
        hi = P.num_q_tiles;  // first segment starting after tend
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (seg_start(mid) > tend) hi = mid; else lo = mid + 1;
        }
        nsteps = tend >= tbeg ? lo - seg0 : 0;
    }
    // rows [t0, t1] of slice i (t1 - t0 < 128; empty for an entry out of range,
    // whose rows are then all invisible)
    auto slice = [&](int i, int &t0, int &t1) {
        if (!SEG) {
            t0 = tbeg + i * BM;
            t1 = min(t0 + BM - 1, tend);
            return;
        }
        int a, n;
        if (!q_segment(P.q_tiles, P.q_tile_rows, seg0 + i, P.Tq, a, n)) {
            t0 = tbeg;
            t1 = tbeg - 1;
            return;
        }
        t0 = max(a, tbeg);
        t1 = min(a + n - 1, tend);
        if (t1 < t0) { t0 = tbeg; t1 = tbeg - 1; }
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NBARS; ++i) mbar_init(&bars[i], 1);
        mbar_init(bar_ptf, EW_THREADS);
        mbar_init(bar_dpr, EW_THREADS);
        mbar_init(bar_dsf, EW_THREADS);
        mbar_init(bar_dqe, EW_THREADS);
        mbar_init(bar_stg, EW_THREADS);
        *abort = status_bad() ? 1 : 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool skip = *abort != 0;
    // region of S^T_i / P^T_i / dQ_i (i even: R0); dP^T_i takes region(i + 1)
    auto region = [&](int i) -> uint32_t { return (i & 1) ? C::T_R1 : C::T_R0; };

    if (warp == 0) {
        // ------------------------------------------------------ producer --
        // K, V, Q_0..Q_2 and dO_0, dO_1 first; then per step i: once dQ_i is
        // staged over the slots of Q_i and dO_i, its reduce-adds into the
        // accumulator rows (b, h, tbeg + 128 i + r) -- rows past the slice's end
        // add zeros (their dS is 0), rows past the tensor's last row are clipped
        // by the tensor map -- and, once they have read the slots, dO_{i+2} and
        // Q_{i+3} into them
        if (lane == 0 && !skip) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_do);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_dq);
            mbar_expect_tx(bar_kv, 2 * C::KT);
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
                tma_load_5d(smem + C::OFF_K + cb * BN * 128, &tm_k, bar_kv, cb * 64, h, ks, 0, b);
                tma_load_5d(smem + C::OFF_V + cb * BN * 128, &tm_v, bar_kv, cb * 64, h, ks, 0, b);
            }
            auto load = [&](bool is_do, int i) {
                uint64_t *bar = is_do ? bar_of + i % OSL : bar_qf + i % QSL;
                uint8_t *dst = smem + (is_do ? C::do_off(i) : C::q_off(i));
                int t0, t1;
                slice(i, t0, t1);
                mbar_expect_tx(bar, C::QT);
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_4d(dst + cb * BM * 128, is_do ? &tm_do : &tm_q, bar, cb * 64, h, t0, b);
            };
            int q_issued = 0, o_issued = 0;
            for (; q_issued < QSL && q_issued < nsteps; ++q_issued) load(false, q_issued);
            for (; o_issued < OSL && o_issued < nsteps; ++o_issued) load(true, o_issued);
            for (int i = 0; i < nsteps; ++i) {
                if (!mbar_wait(bar_stg, i & 1, abort)) break;
                int t0, t1;
                slice(i, t0, t1);
                const int row0 = (b * P.H + h) * P.Tq + t0;
                // the boxes over dO_i's slot as one bulk group, then those over Q_i's:
                // dO_{i+2}, needed first, goes in as soon as its slot has been read
#pragma unroll
                for (int bx = C::NBOX / 2; bx < C::NBOX; ++bx)
                    tma_reduce_add_2d(&tm_dq, smem + C::box_off(i, bx), bx * DQ_BOX_COLS, row0);
                bulk_commit();
#pragma unroll
                for (int bx = 0; bx < C::NBOX / 2; ++bx)
                    tma_reduce_add_2d(&tm_dq, smem + C::box_off(i, bx), bx * DQ_BOX_COLS, row0);
                bulk_commit();
                if (i + OSL < nsteps) {
                    bulk_wait_read_but_newest();  // dO_i's slot is free again
                    load(true, o_issued++);
                }
                if (i + QSL < nsteps) {
                    bulk_wait_read_all();  // and Q_i's
                    load(false, q_issued++);
                }
            }
            bulk_wait_all();  // every reduce-add has landed
            if (*abort) {
                drain_wait(bar_kv, 0);
                for (int i = (q_issued > QSL ? q_issued - QSL : 0); i < q_issued; ++i)
                    drain_wait(bar_qf + i % QSL, (i / QSL) & 1);
                for (int i = (o_issued > OSL ? o_issued - OSL : 0); i < o_issued; ++i)
                    drain_wait(bar_of + i % OSL, (i / OSL) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA ---
        if (lane == 0 && !skip) {
            const uint32_t id_st = idesc_bf16(BN, BM, false);      // M = 128 keys, N = 128 rows
            const uint32_t id_acc = idesc_bf16(BN, D, true);       // M = 128 keys, N = D, B MN-major
            const uint32_t id_dq = idesc_bf16(BM, D, true, true);  // M = 128 rows, N = D, A, B MN-major
            const uint32_t base = smem_u32(smem);
            const uint32_t k_s = base + C::OFF_K, v_s = base + C::OFF_V;
            bool ok = mbar_wait(bar_kv, 0, abort);
            // S^T_i = K Q_i^T into region(i) (waits for Q_i)
            auto issue_st = [&](int i) -> bool {
                if (!mbar_wait(bar_qf + i % QSL, (i / QSL) & 1, abort)) return false;
                tc_fence_after();
                const uint32_t q_s = base + C::q_off(i);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
                    umma_ss(tmem + region(i), sdesc_sw128(k_s + off, 16, 1024),
                            sdesc_sw128(q_s + off, 16, 1024), id_st, kk > 0);
                }
                umma_commit(bar_sf);
                return true;
            };
            // dP^T_i = V dO_i^T into region(i + 1) (waits for dO_i)
            auto issue_dpt = [&](int i) -> bool {
                if (!mbar_wait(bar_of + i % OSL, (i / OSL) & 1, abort)) return false;
                tc_fence_after();
                const uint32_t do_s = base + C::do_off(i);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
                    umma_ss(tmem + region(i + 1), sdesc_sw128(v_s + off, 16, 1024),
                            sdesc_sw128(do_s + off, 16, 1024), id_st, kk > 0);
                }
                umma_commit(bar_dpf);
                return true;
            };
            // dV += P^T_i dO_i: P^T_i rows [32g, 32g + 32) packed into columns
            // [32g, 32g + 16) of region(i)
            auto issue_dv = [&](int i) -> bool {
                if (!mbar_wait(bar_ptf, i & 1, abort)) return false;
                tc_fence_after();
                const uint32_t do_s = base + C::do_off(i);
#pragma unroll
                for (int kk = 0; kk < BM / 16; ++kk)
                    umma_ts(tmem + C::T_DV, tmem + region(i) + (kk >> 1) * 32 + (kk & 1) * 8,
                            sdesc_sw128(do_s + kk * 2048, BM * 128, 1024), id_acc,
                            (i > 0 || kk > 0) ? 1u : 0u);
                umma_commit(bar_dvd);
                return true;
            };
            // dK += dS^T_i Q_i (dS^T K-major) and dQ_i = dS_i K into region(i)
            // (dS MN-major: the same tile; K MN-major), after dV_i read P^T_i there
            auto issue_dk_dq = [&](int i) {
                const uint32_t q_s = base + C::q_off(i), ds_s = base + C::ds_off(i);
#pragma unroll
                for (int kk = 0; kk < BM / 16; ++kk)
                    umma_ss(tmem + C::T_DK,
                            sdesc_sw128(ds_s + (kk >> 2) * (BN * 128) + (kk & 3) * 32, 16, 1024),
                            sdesc_sw128(q_s + kk * 2048, BM * 128, 1024), id_acc,
                            (i > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    umma_ss(tmem + region(i), sdesc_sw128(ds_s + kk * 2048, BN * 128, 1024),
                            sdesc_sw128(k_s + kk * 2048, BN * 128, 1024), id_dq, kk > 0 ? 1u : 0u);
                umma_commit(bar_dqf);
            };
            // Per step i the pipe runs S^T_{i+1}, dK_i + dQ_i, dV_{i+1}, dP^T_{i+1}:
            // S^T_{i+1} overwrites dP^T_i as soon as the element-wise warps have read
            // it (they form and store dS^T_i meanwhile), and dV_{i+1} runs while they
            // read dQ_i out of the region dP^T_{i+1} takes next.
            if (ok && nsteps > 0) {
                ok = issue_st(0);
                if (ok) ok = issue_dpt(0);
                if (ok) ok = issue_dv(0);
                for (int i = 0; ok && i < nsteps; ++i) {
                    ok = mbar_wait(bar_dpr, i & 1, abort);
                    if (!ok) break;
                    tc_fence_after();
                    if (i + 1 < nsteps) ok = issue_st(i + 1);
                    if (ok) ok = mbar_wait(bar_dsf, i & 1, abort);
                    if (!ok) break;
                    tc_fence_after();
                    issue_dk_dq(i);
                    if (i + 1 < nsteps) {
                        // dV_{i+1} reads dO_{i+1}, which no product has waited for yet
                        ok = mbar_wait(bar_of + (i + 1) % OSL, ((i + 1) / OSL) & 1, abort);
                        if (ok) ok = issue_dv(i + 1);
                        if (ok) ok = mbar_wait(bar_dqe, i & 1, abort);
                        if (ok) ok = issue_dpt(i + 1);
                    }
                }
            }
            umma_commit(bar_done);
            drain_wait(bar_done, 0);
        }
    } else {
        // ----------------------------------------------------- element-wise --
        // S^T / dP^T: thread = (key = TMEM lane, quarter eg of a step's rows);
        // dQ_i: thread = (row of the slice = TMEM lane, quarter eg of D)
        const int quad = warp & 3;
        const int eg = (warp - 2) >> 2;
        const int sl = quad * 32 + lane;   // TMEM lane
        const int s = ks + sl;             // local key index
        const int tid = threadIdx.x - 64;  // 0 .. EW_THREADS-1
        const float sl2 = P.scale * 1.4426950408889634f;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        constexpr int HC = BM / EW;  // rows per thread and step
        constexpr int DC = D / EW;   // dQ columns per thread
        // the query rows that see key s: one interval (empty for keys past Tk)
        int ta, tb;
        key_rows(P.mask, s, ta, tb);
        // Row data of step j in slot j & 1: lse and D_t of its rows and the rows
        // [t0, t1] themselves.  Threads 0..127 fill a step's slot one step ahead with
        // asynchronous copies, so no thread waits on a global load inside the loop.
        struct RowSlot {
            float lse[BM], d[BM];
            int t0, t1, pad[2];
        };
        static_assert(sizeof(RowSlot) == C::ROW_BYTES, "row slot layout");
        RowSlot *slots = reinterpret_cast<RowSlot *>(smem + C::OFF_ROW);
        auto prefetch = [&](int j) {
            if (tid >= BM || j >= nsteps) return;
            RowSlot &rs = slots[j & 1];
            int t0, t1;
            slice(j, t0, t1);
            const int t = t0 + tid;
            if (t <= t1) {
                const int64_t o = ((int64_t)b * P.H + h) * P.Tq + t;
                cp_async_4(&rs.lse[tid], lse + o);
                cp_async_4(&rs.d[tid], Dws + o);
                cp_async_commit();
            } else {  // a row past the slice: never visible, D_t must stay finite
                rs.lse[tid] = 0.f;
                rs.d[tid] = 0.f;
            }
            if (tid == 0) {
                rs.t0 = t0;
                rs.t1 = t1;
            }
        };
        // dQ_j: TMEM -> registers -> the swizzled boxes of tm_dq over the slots
        // of Q_j and dO_j (no product reads them once dQ_j is complete); the
        // producer adds them into the accumulator
        auto write_dq = [&](int j) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait(bar_dqf, j & 1, abort))) return false;
            tc_fence_after();
            uint32_t a[DC];
            tmem_ldn<DC>(tl + region(j) + eg * DC, a);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(bar_dqe);  // region(j) may take dP^T_{j+1}
#pragma unroll
            for (int c = 0; c < DC / 4; ++c) {
                const int col = eg * DC + 4 * c;
                const int ch = (col % DQ_BOX_COLS) / 4;
                uint8_t *dst = smem + C::box_off(j, col / DQ_BOX_COLS) + sl * 128 +
                               ((ch ^ (sl & 7)) << 4);
                *reinterpret_cast<uint4 *>(dst) =
                    make_uint4(a[4 * c], a[4 * c + 1], a[4 * c + 2], a[4 * c + 3]);
            }
            fence_proxy_async_smem();  // visible to the TMA unit
            mbar_arrive(bar_stg);
            return true;
        };
        prefetch(0);
        bool ok = !skip;
        for (int i = 0; i < nsteps; ++i) {
            cp_async_wait_all();  // this thread's copies into slot i & 1 have landed
            // Slot i & 1 complete and visible, every thread done with step i-1 (whose
            // slot the next prefetch overwrites), and all element-wise warps agree to go
            // on.  A warp whose wait fails below skips to the next iteration, where
            // every warp stops here (the only named barrier of an iteration).
            ok = group_all(ok);
            if (!ok) break;
            prefetch(i + 1);
            const RowSlot &rs = slots[i & 1];
            // this thread's rows: tr0 .. tr0 + HC - 1, visible while in [ta, tmax]
            const int tr0 = rs.t0 + eg * HC;
            const int tmax = min(tb, rs.t1);
            // ---- P^T_i = exp(S^T_i scale - lse) over region(i)
            ok = __all_sync(0xffffffffu, mbar_wait(bar_sf, i & 1, abort));
            if (!ok) continue;
            tc_fence_after();
            uint32_t v[HC];
            tmem_ldn<HC>(tl + region(i) + eg * HC, v);
            tmem_ld_wait();
            const float *cl = rs.lse + eg * HC;
            float p[HC];
            if (ta <= tr0 && tr0 + HC - 1 <= tmax) {
#pragma unroll
                for (int r = 0; r < HC; ++r)
                    p[r] = ex2(fmaf(__uint_as_float(v[r]), sl2, -1.4426950408889634f * cl[r]));
            } else {
                // a visible row has a finite lse; the others take 0 without using theirs
#pragma unroll
                for (int r = 0; r < HC; ++r) {
                    const bool vis = ta <= tr0 + r && tr0 + r <= tmax;
                    const float e = ex2(fmaf(__uint_as_float(v[r]), sl2, -1.4426950408889634f * cl[r]));
                    p[r] = vis ? e : 0.f;
                }
            }
            {
                uint32_t pk[HC / 2];
#pragma unroll
                for (int c = 0; c < HC / 2; ++c) pk[c] = pack_bf16(p[2 * c], p[2 * c + 1]);
                tmem_stn<HC / 2>(tl + region(i) + eg * HC, pk);
                tmem_st_wait();
            }
            tc_fence_before();
            mbar_arrive(bar_ptf);
            // ---- dQ_{i-1} out
            if (i > 0) {
                ok = write_dq(i - 1);
                if (!ok) continue;
            }
            // ---- dS^T_i = P^T_i (dP^T_i - D) into the shared tile
            ok = __all_sync(0xffffffffu, mbar_wait(bar_dpf, i & 1, abort));
            if (!ok) continue;
            tc_fence_after();
            tmem_ldn<HC>(tl + region(i + 1) + eg * HC, v);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(bar_dpr);  // region(i + 1) may take S^T_{i+1}
            const float *cd = rs.d + eg * HC;
#pragma unroll
            for (int r = 0; r < HC; ++r) p[r] = p[r] * (__uint_as_float(v[r]) - cd[r]);
            // at D = 128 the tile is dO_i's slot: dV_i must have read it
            if (C::DS_IN_DO) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar_dvd, i & 1, abort));
                if (!ok) continue;
            }
            uint8_t *ds_tile = smem + C::ds_off(i);
            // key sl, rows [eg * HC, eg * HC + HC): 16-byte chunks eg * 4 .. eg * 4 + 3
            // of the key's 256-byte row of the swizzled tile
#pragma unroll
            for (int j = 0; j < HC / 8; ++j) {
                uint4 u;
                u.x = pack_bf16(p[8 * j + 0], p[8 * j + 1]);
                u.y = pack_bf16(p[8 * j + 2], p[8 * j + 3]);
                u.z = pack_bf16(p[8 * j + 4], p[8 * j + 5]);
                u.w = pack_bf16(p[8 * j + 6], p[8 * j + 7]);
                *reinterpret_cast<uint4 *>(ds_tile + sw128_offset(sl, eg * (HC / 8) + j, BN)) = u;
            }
            fence_proxy_async_smem();  // dS^T_i visible to the tensor pipe
            mbar_arrive(bar_dsf);
        }
        cp_async_wait_all();  // no copy outlives the loop
        if (ok && nsteps > 0) ok = write_dq(nsteps - 1);
        // ------------------------------------------------------ epilogue ---
        // each warpgroup writes a quarter of the D columns of its keys' dV and dK
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, abort));
        tc_fence_after();
        constexpr int NCH = D / 16 / EW;  // 16-column chunks per warpgroup
#pragma unroll 1
        for (int q = 0; q < 2 * NCH; ++q) {  // dV chunks, then dK chunks
            const int c = eg * NCH + (q % NCH);
            const bool is_k = q >= NCH;
            uint32_t a[16];
            if (ok && nsteps > 0) {
                tmem_ldn<16>(tl + (is_k ? C::T_DK : C::T_DV) + c * 16, a);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) a[e] = 0u;
            }
            if (ok && s < P.Tk) {
                const int64_t off = b * P.kv_sb + (int64_t)s * P.kv_st + (int64_t)h * D + c * 16;
                grad_out16(P, is_k ? dk : dv, off, reinterpret_cast<const float *>(a),
                           is_k ? P.scale : 1.f);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace kvq
}  // namespace tcbwd

constexpr bool kTcBwdAvailable = true;

inline bool tc_bwd_shape_ok(const eagle_attn_params *p) {
    return p->num_blocks - 1 <= tcbwd::MAX_DIAG;
}

}  // namespace eagle
