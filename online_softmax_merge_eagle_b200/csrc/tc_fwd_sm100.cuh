// tc_fwd_sm100.cuh -- tensor-core forward of the joint softmax for sm_100a.
//
// One CTA owns a 128-row query tile of one (b, h).  Every MMA reads its A
// operand from tensor memory: Q is copied into TMEM once (tcgen05.cp from the
// shared tile, bf16 pairs, one row per lane), so S = Q K^T is a TMEM x SMEM
// product like O += P V, with P written over the S it came from; shared memory
// holds the Q tile (the source of that copy) and a five-slot K/V ring.
// Warp roles:
//   warp 0     TMA producer: Q once, then the block-0 K and V tiles of 128 keys
//              as separate items of a ring of [128 x D] slots (128-byte
//              swizzled, as the MMA reads them), then the diagonal blocks' K_i /
//              V_i tiles of the same 128 rows through the same ring;
//   warp 1     TMEM owner and MMA issuer (one thread): S_j = Q K_j^T into one of
//              two TMEM S buffers, O += P_j V_j into the TMEM O buffer, S_{j+1}
//              issued ahead of PV_j; after the last PV, Q K_i^T for every
//              diagonal block i through the same S buffers (its diagonal holds
//              the rows' logits q_t . k_i_t);
//   warps 2-9  softmax, two warpgroups, each one query row per thread (TMEM
//              lane = row) and half of the key columns: S from TMEM, per-row
//              interval mask, running max / sum in the exp2 domain with a
//              reference max that only moves when a row's max grows by more than
//              2^8 (O rescaled in TMEM then, rarely), P as bf16 written back over
//              the S columns it came from; then the epilogue, which folds the
//              NB-1 diagonal logits (q_t . k_i_t) * scale (each row's diagonal
//              element of Q K_i^T, from TMEM) and values v_i_t (read from the
//              ring) into (m, l, O) by the same online update, normalises once
//              and writes out and lse.
// NeMo AutoModel "eagle.ring_attention", _CachedRingAttention (the joint
// softmax), _update_out_and_lse / _merge_diag (the online merge it folds).
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace eagle {
namespace tcfwd {

using namespace sm100;

constexpr int BM = 128;       // query rows per CTA (TMEM lanes)
constexpr int BN = 128;       // keys per tile
constexpr int EW = 2;         // softmax warpgroups: each owns half the columns of every row
constexpr int EW_THREADS = 128 * EW;
constexpr int THREADS = 64 + EW_THREADS;
constexpr float RESCALE_LOG2 = 8.f;  // the reference max moves when the max grows by > 2^8
template <int D>
struct Cfg {
    static constexpr int TILE = BM * D * 2;  // bytes of a [128 x D] bf16 tile
    static constexpr int KSTEPS = D / 16;    // MMA K steps of QK^T
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_XCH = OFF_Q + TILE;  // row-max exchange [2][EW][BM], l [EW][BM]
    static constexpr int XCH_BYTES = (2 * EW + EW) * BM * 4;
    static constexpr int NBARS = 32;
    static constexpr int BAR_BYTES = NBARS * 8 + 16;
    // Ring of [128 x D] tiles: the items K_0, V_0, K_1, V_1, ... each take one
    // slot, so a K tile (released after its S MMA) frees its slot long before
    // the V tile of the same keys; as many slots as the 227 KB allow (at most 8).
    static constexpr int FREE = 232448 - 1024 - TILE - XCH_BYTES - BAR_BYTES;
    static constexpr int SLOTS = FREE / TILE < 8 ? FREE / TILE : 8;
    static_assert(SLOTS >= 4, "ring too shallow");
    static constexpr int OFF_RING = ((OFF_XCH + XCH_BYTES + 1023) / 1024) * 1024;
    static constexpr int OFF_BAR = OFF_RING + SLOTS * TILE;
    static constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
    static_assert(SMEM <= 232448, "shared memory");
    // S0, S1 (128 columns each), O (D columns), Q (D / 2 columns of bf16 pairs)
    static constexpr uint32_t TMEM_S0 = 0, TMEM_S1 = 128, TMEM_O = 256, TMEM_Q = 384,
                              TMEM_COLS = 512;
    static_assert(TMEM_O + D <= TMEM_Q && TMEM_Q + D / 2 <= TMEM_COLS, "TMEM budget");
};

// Barrier of the softmax warps (named barrier 1) that also ANDs `v` over them,
// so that every warp takes the same exit decision.
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

// Barrier of the two softmax warps that share TMEM lanes quad * 32 .. + 31 (one per
// warpgroup; named barrier 2 + quad, 64 threads) that also ANDs `v` over them.
__device__ __forceinline__ bool pair_all(bool v, int quad) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, 64, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(2 + quad)
        : "memory");
    return r != 0;
}

// Bounded wait used only while draining after an abort (ignores the abort flag).
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > 100000000ull) return;
}

template <typename TO>
__device__ __forceinline__ void store_chunk32(TO *dst, const float (&v)[32], float inv);
template <>
__device__ __forceinline__ void store_chunk32<__nv_bfloat16>(__nv_bfloat16 *dst,
                                                             const float (&v)[32], float inv) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 u;
        u.x = pack_bf16(v[c * 8 + 0] * inv, v[c * 8 + 1] * inv);
        u.y = pack_bf16(v[c * 8 + 2] * inv, v[c * 8 + 3] * inv);
        u.z = pack_bf16(v[c * 8 + 4] * inv, v[c * 8 + 5] * inv);
        u.w = pack_bf16(v[c * 8 + 6] * inv, v[c * 8 + 7] * inv);
        reinterpret_cast<uint4 *>(dst)[c] = u;
    }
}
template <>
__device__ __forceinline__ void store_chunk32<float>(float *dst, const float (&v)[32], float inv) {
#pragma unroll
    for (int c = 0; c < 8; ++c)
        reinterpret_cast<float4 *>(dst)[c] =
            make_float4(v[c * 4] * inv, v[c * 4 + 1] * inv, v[c * 4 + 2] * inv, v[c * 4 + 3] * inv);
}

template <int D, typename TO>
__global__ void __launch_bounds__(THREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const Problem P, TO *__restrict__ out,
               float *__restrict__ lse_out) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = (uint64_t *)(smem + C::OFF_BAR);
    uint64_t *bar_q = bars + 0;                  // Q tile landed in shared memory
    uint64_t *bar_full = bars + 1;               // [slot]: ring item landed
    uint64_t *bar_empty = bar_full + C::SLOTS;   // [slot]: ring item consumed
    uint64_t *bar_sf = bar_empty + C::SLOTS;     // [2]: S_j in TMEM buffer j & 1
    // [2]: P_j written (EW_THREADS arrivals), tile j on barrier j & 1: the P of
    // tile j + 2 needs S_{j+2}, issued only after PV_j, so the MMA issuer's wait
    // for P_j can never find its barrier two phases on
    uint64_t *bar_pf = bar_sf + 2;
    uint64_t *bar_od = bar_pf + 2;               // PV_j complete
    uint64_t *bar_fin = bar_od + 1;              // MMA issuer: everything issued has completed
    uint64_t *bar_sc = bar_fin + 1;              // [2]: diagonal item d's S read (EW_THREADS arrivals)
    static_assert(C::NBARS >= 1 + 2 * C::SLOTS + 8, "barrier slots");
    uint32_t *tmem_slot = (uint32_t *)(bars + C::NBARS);
    volatile int *abort = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_qtiles = (P.Tq + BM - 1) / BM;
    // heaviest causal tiles first, or the caller's tile / segment list (its
    // order): rows [t0, t0 + nrows) of the tile, nrows <= 128
    int t0 = (n_qtiles - 1 - (int)blockIdx.x) * BM, nrows = min(BM, P.Tq - t0);
    if (P.q_tiles && !q_segment(P.q_tiles, P.q_tile_rows, blockIdx.x, P.Tq, t0, nrows)) {
        if (threadIdx.x == 0) raise_status(EAGLE_ATTN_DEV_BAD_TILE);  // CTA-uniform: nothing
        return;                                                       // allocated yet
    }
    const int h = blockIdx.y, b = blockIdx.z;

    int kbeg, kend;
    rows_key_range(P.mask, t0, t0 + nrows - 1, kbeg, kend);
    const int ntiles = kend >= kbeg ? (kend - kbeg + BN) / BN : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NBARS; ++i) mbar_init(&bars[i], 1);
        mbar_init(bar_pf, EW_THREADS);
        mbar_init(bar_pf + 1, EW_THREADS);
        mbar_init(bar_sc, EW_THREADS);
        mbar_init(bar_sc + 1, EW_THREADS);
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
    const bool skip = *abort != 0;  // uniform: read after the barrier

    if (warp == 0) {
        // ------------------------------------------------------ producer --
        if (lane == 0 && !skip) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_expect_tx(bar_q, C::TILE);
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb)
                tma_load_4d(smem + C::OFF_Q + cb * BM * 128, &tm_q, bar_q, cb * 64, h, t0, b);
            // ring items: K_j, V_j of the block-0 key tiles, then K_i, V_i of
            // this query tile's rows for every diagonal block i = 1 .. NB-1
            const int n_tiles = ntiles + P.NB - 1;
            int issued = 0;
            bool go = true;
            for (int it = 0; go && it < n_tiles; ++it) {
                const int row = it < ntiles ? kbeg + it * BN : t0;
                const int blk = it < ntiles ? 0 : it - ntiles + 1;
#pragma unroll
                for (int kv = 0; kv < 2; ++kv) {
                    const int n = 2 * it + kv;
                    const int sl = n % C::SLOTS;
                    if (!mbar_wait(bar_empty + sl, ((n / C::SLOTS) & 1) ^ 1, abort)) {
                        go = false;
                        break;
                    }
                    mbar_expect_tx(bar_full + sl, C::TILE);
#pragma unroll
                    for (int cb = 0; cb < D / 64; ++cb)
                        tma_load_5d(smem + C::OFF_RING + sl * C::TILE + cb * BN * 128,
                                    kv ? &tm_v : &tm_k, bar_full + sl, cb * 64, h, row, blk, b);
                    issued = n + 1;
                }
            }
            if (*abort) {
                // let every copy this thread started land before the CTA exits
                drain_wait(bar_q, 0);
                for (int n = (issued > C::SLOTS ? issued - C::SLOTS : 0); n < issued; ++n)
                    drain_wait(bar_full + n % C::SLOTS, (n / C::SLOTS) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA ---
        if (lane == 0 && !skip) {
            const uint32_t id_qk = idesc_bf16(BM, BN, false);
            const uint32_t id_pv = idesc_bf16(BM, D, true);
            const uint32_t ring = smem_u32(smem + C::OFF_RING);
            const uint32_t qs = smem_u32(smem + C::OFF_Q);
            bool ok = mbar_wait(bar_q, 0, abort);
            if (ok) {
                // Q into TMEM, K step kk (16 columns of the tile) into TMEM
                // columns 8kk .. 8kk+7; the MMAs below run after these copies
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C::KSTEPS; ++kk)
                    tmem_cp_128x256b(tmem + C::TMEM_Q + kk * 8,
                                     sdesc_sw128(qs + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16,
                                                 1024));
            }
            // S_j = Q K_j^T with Q from TMEM (bf16 pairs: K step kk = columns 8kk .. 8kk+7)
            auto issue_s = [&](int j) -> bool {
                const int n = 2 * j, sl = n % C::SLOTS;
                if (!mbar_wait(bar_full + sl, (n / C::SLOTS) & 1, abort)) return false;
                tc_fence_after();
                const uint32_t d = tmem + ((j & 1) ? C::TMEM_S1 : C::TMEM_S0);
#pragma unroll
                for (int kk = 0; kk < C::KSTEPS; ++kk) {
                    const uint32_t koff = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
                    umma_ts(d, tmem + C::TMEM_Q + kk * 8,
                            sdesc_sw128(ring + sl * C::TILE + koff, 16, 1024), id_qk, kk > 0);
                }
                umma_commit(bar_sf + (j & 1));
                umma_commit(bar_empty + sl);
                return true;
            };
            // O += P_j V_j; P_j lives in the S buffer it replaced: keys
            // [64g, 64g + 64) of warpgroup g packed into columns [64g, 64g + 32)
            auto issue_pv = [&](int j) -> bool {
                const int n = 2 * j + 1, sl = n % C::SLOTS;
                if (!mbar_wait(bar_pf + (j & 1), (j >> 1) & 1, abort)) return false;
                if (!mbar_wait(bar_full + sl, (n / C::SLOTS) & 1, abort)) return false;
                tc_fence_after();
                const uint32_t pa = tmem + ((j & 1) ? C::TMEM_S1 : C::TMEM_S0);
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    umma_ts(tmem + C::TMEM_O, pa + (kk >> 2) * (BN / EW) + (kk & 3) * 8,
                            sdesc_sw128(ring + sl * C::TILE + kk * 2048, BN * 128, 1024), id_pv,
                            (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(bar_empty + sl);
                umma_commit(bar_od);
                return true;
            };
            if (ok && ntiles > 0) {
                ok = issue_s(0);
                for (int j = 0; ok && j < ntiles; ++j) {
                    if (j + 1 < ntiles) ok = issue_s(j + 1);
                    if (ok) ok = issue_pv(j);
                }
            }
            // diagonal blocks: item d (block d + 1) continues the S sequence as
            // j = ntiles + d, with K_{d+1} from the ring.  Its S buffer was last
            // used by item j - 2: a block-0 tile, whose PV (issued earlier) runs
            // first, or item d - 2, whose diagonal the softmax warps have read.
            for (int d = 0; ok && d + 1 < P.NB; ++d) {
                if (d >= 2) ok = mbar_wait(bar_sc + (d & 1), ((d - 2) >> 1) & 1, abort);
                if (ok) ok = issue_s(ntiles + d);
            }
            umma_commit(bar_fin);
            drain_wait(bar_fin, 0);
        }
    } else {
        // ------------------------------------------------------ softmax ---
        // thread = (row = TMEM lane, half of the columns); the two halves of a
        // row agree on the running max through shared memory once per tile, the
        // two warps of those rows meeting at their own named barrier
        const int quad = warp & 3;
        const int eg = (warp - 2) >> 2;
        const int r = quad * 32 + lane;
        const int t = t0 + r;
        const bool row_ok = r < nrows;  // a row of this tile (the rest: other rows, or past Tq)
        constexpr int HC = BN / EW;  // 64 key columns per thread and tile
        int lo = 1, hi = 0;
        if (row_ok && row_interval(P.mask, t, lo, hi) != 0) { lo = 1; hi = 0; }
        const float sl2 = P.scale * 1.4426950408889634f;
        // m: reference max (exp2 domain) of l and O; -inf until the row sees a key
        float m = -INFINITY, l = 0.f;  // l: this half's partial sum
        float *xmax = reinterpret_cast<float *>(smem + C::OFF_XCH);  // [2][EW][BM]
        float *xsum = xmax + 2 * EW * BM;                             // [EW][BM]
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        bool ok = !skip;
        for (int j = 0; j < ntiles; ++j) {
            const int ks = kbeg + j * BN + eg * HC;  // first key of this half
            const uint32_t sb = tl + ((j & 1) ? C::TMEM_S1 : C::TMEM_S0) + eg * HC;
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_sf + (j & 1), (j >> 1) & 1, abort));
            uint32_t s[HC];
            float mx = -INFINITY;
            if (ok) {
                tc_fence_after();
                tmem_ld32(sb, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
                tmem_ld32(sb + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
                tmem_ld_wait();
                if (!__all_sync(0xffffffffu, lo <= ks && ks + HC - 1 <= hi)) {
#pragma unroll
                    for (int c = 0; c < HC; ++c)
                        if (ks + c < lo || ks + c > hi) s[c] = __float_as_uint(-INFINITY);
                }
                float mx0 = __uint_as_float(s[0]), mx1 = __uint_as_float(s[1]);
                float mx2 = __uint_as_float(s[2]), mx3 = __uint_as_float(s[3]);
#pragma unroll
                for (int c = 4; c < HC; c += 4) {
                    mx0 = fmaxf(mx0, __uint_as_float(s[c]));
                    mx1 = fmaxf(mx1, __uint_as_float(s[c + 1]));
                    mx2 = fmaxf(mx2, __uint_as_float(s[c + 2]));
                    mx3 = fmaxf(mx3, __uint_as_float(s[c + 3]));
                }
                mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
                xmax[((j & 1) * EW + eg) * BM + r] = mx;
            }
            // both halves of these rows have their maxima in shared memory (the other
            // rows' warps need not wait for it)
            ok = pair_all(ok, quad);
            if (!ok) break;
#pragma unroll
            for (int g = 0; g < EW; ++g) mx = fmaxf(mx, xmax[((j & 1) * EW + g) * BM + r]);
            // move the reference only when the max grew by more than 2^8 (or the
            // row saw its first key): P <= 2^8 stays exact enough in bf16
            const float mt = mx * sl2;
            float alpha = 1.f;
            if (mt > m + RESCALE_LOG2) {
                alpha = ex2(m - mt);  // 0 while m = -inf: l and O are 0 then
                m = mt;
            }
            const float m_use = (m == -INFINITY) ? 0.f : m;
            float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
            for (int c = 0; c < HC; c += 2) {
                const float p0 = ex2(fmaf(__uint_as_float(s[c]), sl2, -m_use));
                const float p1 = ex2(fmaf(__uint_as_float(s[c + 1]), sl2, -m_use));
                sum0 += p0;
                sum1 += p1;
                s[c / 2] = pack_bf16(p0, p1);
            }
            if (j > 0 && __any_sync(0xffffffffu, alpha < 1.f)) {
                // PV_{j-1} done: O is stable (S_j complete implies PV_{j-2} is)
                ok = __all_sync(0xffffffffu, mbar_wait(bar_od, (j - 1) & 1, abort));
                if (!ok) continue;
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < D / 32 / EW; ++c) {
                    const uint32_t oc = tl + C::TMEM_O + (eg * (D / 32 / EW) + c) * 32;
                    uint32_t o[32];
                    tmem_ld32(oc, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(oc, o);
                }
            }
            // P (bf16 pairs) over the first half of this warpgroup's S columns
            tmem_st32(sb, *reinterpret_cast<const uint32_t(*)[32]>(&s[0]));
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bar_pf + (j & 1));
            l = l * alpha + (sum0 + sum1);
        }
        // ------------------------------------------------------- epilogue --
        // diagonal blocks: an online (m_d, l_d, acc) over the NB-1 one-key blocks
        // of this row.  The logit q_t . k_i_t is the row's diagonal element of
        // Q K_i^T, which the MMA issuer computes into the S buffers (thread
        // lane l of quad w reads columns 32w .. 32w+31 and keeps element l);
        // V_i comes from the ring, each warpgroup accumulating its half of the
        // value columns.
        constexpr int NCH = D / 32 / EW;
        float acc[NCH * 32];
#pragma unroll
        for (int i = 0; i < NCH * 32; ++i) acc[i] = 0.f;
        float m_d = -INFINITY, l_d = 0.f;
        for (int i = 1; i < P.NB; ++i) {
            const int dix = i - 1, u = ntiles + dix;
            const int nv = 2 * u + 1, slv = nv % C::SLOTS;
            float zq = 0.f;
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_sf + (u & 1), (u >> 1) & 1, abort));
            if (ok) {
                tc_fence_after();
                uint32_t sv[32];
                tmem_ld32(tl + ((u & 1) ? C::TMEM_S1 : C::TMEM_S0) + quad * 32, sv);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 32; ++c) zq = (c == lane) ? __uint_as_float(sv[c]) : zq;
            }
            tc_fence_before();
            mbar_arrive(bar_sc + (dix & 1));  // this S buffer may take item i + 2
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_full + slv, (nv / C::SLOTS) & 1, abort));
            if (ok) {
                const uint8_t *vt = smem + C::OFF_RING + slv * C::TILE;
                const float d = zq * sl2;
                const float mn = fmaxf(m_d, d);
                const float sc = ex2(m_d - mn), pd = ex2(d - mn);
                l_d = l_d * sc + pd;
                m_d = mn;
#pragma unroll
                for (int c = 0; c < NCH * 4; ++c) {
                    const uint4 vv = *reinterpret_cast<const uint4 *>(
                        vt + sw128_offset(r, eg * NCH * 4 + c, BM));
                    const uint32_t *pv = &vv.x;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc[c * 8 + 2 * e] =
                            fmaf(acc[c * 8 + 2 * e], sc, pd * __uint_as_float(pv[e] << 16));
                        acc[c * 8 + 2 * e + 1] = fmaf(acc[c * 8 + 2 * e + 1], sc,
                                                      pd * __uint_as_float(pv[e] & 0xffff0000u));
                    }
                }
            }
            ok = group_all(ok);  // every softmax thread is done with this V slot
            if (ok && threadIdx.x == 64) mbar_arrive(bar_empty + slv);
        }
        // everything the MMA issuer started (the last PV included) has completed
        if (ok && ntiles > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar_fin, 0, abort));
            tc_fence_after();
        }
        xsum[eg * BM + r] = l;
        ok = group_all(ok);  // both partial block-0 sums are in shared memory
        float l_blk = 0.f;
#pragma unroll
        for (int g = 0; g < EW; ++g) l_blk += xsum[g * BM + r];
        const float m_fin = fmaxf(m, m_d);
        const float m_use = (m_fin == -INFINITY) ? 0.f : m_fin;
        const float alpha = ex2(m - m_use), beta = ex2(m_d - m_use);
        const float l_fin = l_blk * alpha + l_d * beta;
        const float inv = l_fin > 0.f ? 1.f / l_fin : 0.f;
#pragma unroll
        for (int cc = 0; cc < NCH; ++cc) {
            const int c = eg * NCH + cc;
            uint32_t o[32];
            if (ntiles > 0 && ok) {
                tmem_ld32(tl + C::TMEM_O + c * 32, o);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = 0u;
            }
            float res[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                res[i] = fmaf(__uint_as_float(o[i]), alpha, acc[cc * 32 + i] * beta);
            if (row_ok && ok) {
                TO *orow = out + b * P.q_sb + (int64_t)t * P.q_st + (int64_t)h * D + c * 32;
                store_chunk32<TO>(orow, res, inv);
            }
        }
        if (eg == 0 && row_ok && ok)
            lse_out[((int64_t)b * P.H + h) * P.Tq + t] =
                l_fin > 0.f ? (m_use + __log2f(l_fin)) * 0.6931471805599453f : -INFINITY;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace tcfwd

// ------------------------------------------------------------------ host --
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)ptr;
    }
    return fn;
}

// Tensor map over a bf16 tensor with innermost dim D (element stride 1); box =
// 64 elements x box_rows rows (dim 2), 1 along every other dim; 128 B swizzle.
inline bool make_tmap_bf16(CUtensorMap *m, const void *base, int rank, const uint64_t *dims,
                           const uint64_t *strides_bytes, uint32_t box_rows) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    cuuint64_t gd[5], gs[4];
    cuuint32_t box[5], es[5];
    for (int i = 0; i < rank; ++i) {
        gd[i] = dims[i];
        box[i] = 1;
        es[i] = 1;
    }
    for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
    box[0] = 64;
    box[2] = box_rows;
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base),
                     gd, gs, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D tensor map over a row-major fp32 matrix [rows, cols] (row stride = cols);
// box = box_cols x box_rows with the 128-byte swizzle (box_cols * 4 = 128).
inline bool make_tmap_f32_2d(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                             uint32_t box_cols, uint32_t box_rows) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    cuuint64_t gd[2] = {cols, rows}, gs[1] = {cols * 4};
    cuuint32_t box[2] = {box_cols, box_rows}, es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), gd, gs, box,
                     es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tensor maps of q-like [B, T, H, D] and cache-like [B, NB, T, H, D] operands.
inline bool make_q_tmap(CUtensorMap *m, const void *base, const Problem &P, uint32_t box_rows) {
    const uint64_t dims[4] = {(uint64_t)P.D, (uint64_t)P.H, (uint64_t)P.Tq, (uint64_t)P.B};
    const uint64_t sb = P.B > 1 ? (uint64_t)P.q_sb * 2 : (uint64_t)P.Tq * P.q_st * 2;
    const uint64_t st[3] = {(uint64_t)P.D * 2, (uint64_t)P.q_st * 2, sb ? sb : 16};
    return make_tmap_bf16(m, base, 4, dims, st, box_rows);
}
inline bool make_kv_tmap(CUtensorMap *m, const void *base, const Problem &P, uint32_t box_rows) {
    const uint64_t dims[5] = {(uint64_t)P.D, (uint64_t)P.H, (uint64_t)P.Tk, (uint64_t)P.NB,
                              (uint64_t)P.B};
    uint64_t sblk = P.NB > 1 ? (uint64_t)P.kv_sblk * 2 : (uint64_t)P.Tk * P.kv_st * 2;
    uint64_t sb = P.B > 1 ? (uint64_t)P.kv_sb * 2 : sblk * P.NB;
    const uint64_t st[4] = {(uint64_t)P.D * 2, (uint64_t)P.kv_st * 2, sblk ? sblk : 16,
                            sb ? sb : 16};
    return make_tmap_bf16(m, base, 5, dims, st, box_rows);
}

inline bool tc_fwd_shape_ok(const eagle_attn_params *p) {
    return p->dtype == EAGLE_ATTN_BF16 && (p->D == 64 || p->D == 128) &&
           p->scale > 0.f && p->scale < 1e30f;
}

}  // namespace eagle
