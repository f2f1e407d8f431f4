// eagleattn.cu -- the C ABI of libeagleattn (declared in include/eagleattn.h):
// argument validation, dispatch between the tensor-core (sm_100a tcgen05)
// kernels and the generic CUDA-core kernels, and launches.  One translation
// unit: the kernel headers below are included here.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "generic_attn.cuh"
#include "rowwise.cuh"
#include "tc_fwd_sm100.cuh"
#include "tc_bwd_sm100.cuh"

using namespace eagle;

// Scratch of eagle_attn_bwd_noalloc: a fixed device array, so that callers
// that cannot allocate still get a backward.  Host code must not pass this
// name to a kernel (on the host it is a stand-in, not a device address); the
// device address comes from cudaGetSymbolAddress, per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[EAGLE_ATTN_NOALLOC_SCRATCH_BYTES];

namespace {

std::atomic<uint64_t> g_launches{0};

// Every kernel launch of the library goes through one of these.
inline int after_launch(int n = 1) {
    g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed);
    return cudaGetLastError() == cudaSuccess ? EAGLE_ATTN_OK : EAGLE_ATTN_ERR_CUDA;
}

inline void prof_mark(void *ev, cudaStream_t s) {
    if (ev) cudaEventRecord((cudaEvent_t)ev, s);
}

size_t dtype_size(int dt) { return dt == EAGLE_ATTN_F32 ? 4 : 2; }

bool tc_supported(const eagle_attn_params *p, bool bwd) {
    // empty extents go to the generic kernels (no tensor map of an empty array)
    if (!tc_fwd_shape_ok(p) || p->Tk == 0 || p->Tq == 0) return false;
    return !bwd || (kTcBwdAvailable && tc_bwd_shape_ok(p));
}

bool aligned16(const void *p) { return p == nullptr || ((uintptr_t)p & 15u) == 0; }

struct Resolved {
    Problem P;
    bool tc;  // use the tensor-core kernels
};

// Fills the kernel view of *p; returns an eagle_attn_status.
int resolve(const eagle_attn_params *p, bool bwd, Resolved *r) {
    if (!p) return EAGLE_ATTN_ERR_NULL;
    if (p->struct_size != sizeof(eagle_attn_params) || p->abi_version != EAGLE_ATTN_ABI_VERSION)
        return EAGLE_ATTN_ERR_ABI;
    if (p->dtype != EAGLE_ATTN_F32 && p->dtype != EAGLE_ATTN_BF16) return EAGLE_ATTN_ERR_DTYPE;
    if (p->out_dtype != p->dtype && p->out_dtype != EAGLE_ATTN_F32) return EAGLE_ATTN_ERR_DTYPE;
    if (p->B < 1 || p->Tq < 0 || p->Tk < 0 || p->H < 1 || p->num_blocks < 1)
        return EAGLE_ATTN_ERR_SHAPE;
    if (p->D != 32 && p->D != 64 && p->D != 128) return EAGLE_ATTN_ERR_SHAPE;
    if (p->num_blocks > 1 && p->Tk != p->Tq) return EAGLE_ATTN_ERR_SHAPE;
    if (p->cu_seqlens && (p->B != 1 || p->num_docs < 1)) return EAGLE_ATTN_ERR_VARLEN;
    // buffers of an empty extent may be NULL (an empty torch tensor has no storage)
    const bool rows_ = p->Tq > 0, keys_ = p->Tk > 0;
    if (rows_ && (!p->q || !p->out || !p->lse)) return EAGLE_ATTN_ERR_NULL;
    if (keys_ && (!p->cache_k || !p->cache_v)) return EAGLE_ATTN_ERR_NULL;
    if (bwd && rows_ && (!p->grad_out || !p->dq)) return EAGLE_ATTN_ERR_NULL;
    if (bwd && keys_ && (!p->dk || !p->dv)) return EAGLE_ATTN_ERR_NULL;
    if (p->impl < EAGLE_ATTN_IMPL_AUTO || p->impl > EAGLE_ATTN_IMPL_GENERIC)
        return EAGLE_ATTN_ERR_UNSUPPORTED;
    if (p->grad_mode != EAGLE_ATTN_GRAD_STORE && p->grad_mode != EAGLE_ATTN_GRAD_ACCUMULATE_F32)
        return EAGLE_ATTN_ERR_UNSUPPORTED;

    Problem &P = r->P;
    P.B = p->B; P.Tq = p->Tq; P.Tk = p->Tk; P.H = p->H; P.D = p->D; P.NB = p->num_blocks;
    P.scale = p->scale;
    P.grad_accum = (bwd && p->grad_mode == EAGLE_ATTN_GRAD_ACCUMULATE_F32) ? 1 : 0;
    P.q_tiles = p->q_tiles;
    P.q_tile_rows = p->q_tiles ? p->q_tile_rows : nullptr;
    P.num_q_tiles = p->q_tiles ? p->num_q_tiles : 0;
    if (p->q_tiles && p->num_q_tiles < 0) return EAGLE_ATTN_ERR_SHAPE;
    if (p->q_tile_rows && !p->q_tiles) return EAGLE_ATTN_ERR_SHAPE;
    const int64_t HD = (int64_t)p->H * p->D;
    P.q_st = p->q_stride_t ? p->q_stride_t : HD;
    P.q_sb = p->q_stride_b ? p->q_stride_b : (int64_t)p->Tq * P.q_st;
    P.kv_st = p->kv_stride_t ? p->kv_stride_t : HD;
    P.kv_sblk = p->kv_stride_blk ? p->kv_stride_blk : (int64_t)p->Tk * P.kv_st;
    P.kv_sb = p->kv_stride_b ? p->kv_stride_b : (int64_t)p->num_blocks * P.kv_sblk;
    if (P.q_st < HD || P.kv_st < HD) return EAGLE_ATTN_ERR_STRIDE;
    if (p->B > 1 && P.q_sb < (int64_t)p->Tq * P.q_st) return EAGLE_ATTN_ERR_STRIDE;
    if (p->num_blocks > 1 && P.kv_sblk < (int64_t)p->Tk * P.kv_st) return EAGLE_ATTN_ERR_STRIDE;
    if (p->B > 1 && P.kv_sb < (int64_t)(p->num_blocks - 1) * P.kv_sblk + (int64_t)p->Tk * P.kv_st)
        return EAGLE_ATTN_ERR_STRIDE;
    // 16-byte rows and bases (vector loads, TMA)
    const size_t es = dtype_size(p->dtype);
    if ((P.q_st * es) % 16 || (P.q_sb * es) % 16 || (P.kv_st * es) % 16 || (P.kv_sblk * es) % 16 ||
        (P.kv_sb * es) % 16)
        return EAGLE_ATTN_ERR_ALIGN;
    if (p->out_dtype == EAGLE_ATTN_F32 && ((P.q_st * 4) % 16 || (P.q_sb * 4) % 16))
        return EAGLE_ATTN_ERR_ALIGN;
    if (!aligned16(p->q) || !aligned16(p->cache_k) || !aligned16(p->cache_v) || !aligned16(p->out) ||
        !aligned16(p->lse) || !aligned16(p->grad_out) || !aligned16(p->dq) || !aligned16(p->dk) ||
        !aligned16(p->dv) || !aligned16(p->workspace))
        return EAGLE_ATTN_ERR_ALIGN;

    P.mask.cu = p->cu_seqlens;
    P.mask.num_docs = p->cu_seqlens ? p->num_docs : 0;
    P.mask.q_off = p->q_pos_offset;
    P.mask.k_off = p->k_pos_offset;
    P.mask.causal = p->causal ? 1 : 0;
    P.mask.Tq = p->Tq;
    P.mask.Tk = p->Tk;

    bool tc_ok = tc_supported(p, bwd);
    if (p->impl == EAGLE_ATTN_IMPL_TENSOR_CORE && !tc_ok) return EAGLE_ATTN_ERR_UNSUPPORTED;
    r->tc = (p->impl == EAGLE_ATTN_IMPL_TENSOR_CORE) || (p->impl == EAGLE_ATTN_IMPL_AUTO && tc_ok);
    // fp32 accumulation of the gradients is served by the tensor-core backward only
    if (P.grad_accum && !r->tc) return EAGLE_ATTN_ERR_UNSUPPORTED;
    // so is a query-tile list; in the backward, by the five-product kernel only
    if (P.q_tiles && !r->tc) return EAGLE_ATTN_ERR_UNSUPPORTED;
    if (bwd && P.q_tiles && p->deterministic) return EAGLE_ATTN_ERR_UNSUPPORTED;
    return EAGLE_ATTN_OK;
}

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return EAGLE_ATTN_OK;
    return EAGLE_ATTN_ERR_CUDA;
}

int launch_check_cu(const eagle_attn_params *p, cudaStream_t s) {
    if (!p->cu_seqlens) return EAGLE_ATTN_OK;
    check_cu_kernel<<<1, 256, 0, s>>>(p->cu_seqlens, p->num_docs, p->max_seqlen, p->q_pos_offset,
                                      p->q_pos_offset + p->Tq, p->k_pos_offset,
                                      p->k_pos_offset + p->Tk);
    return after_launch();
}

template <typename T, typename TO, int D>
int generic_fwd_launch(const Problem &P, const eagle_attn_params *p, cudaStream_t s) {
    if (P.Tq == 0) return EAGLE_ATTN_OK;
    auto kern = generic_fwd_kernel<T, TO, D>;
    const int smem = generic_fwd_smem_floats<D>() * 4;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return EAGLE_ATTN_ERR_CUDA;
    dim3 grid((P.Tq + GT - 1) / GT, P.H, P.B);
    prof_mark(p->prof_start, s);
    kern<<<grid, GTHREADS, smem, s>>>(P, (const T *)p->q, (const T *)p->cache_k,
                                       (const T *)p->cache_v, (TO *)p->out, p->lse);
    int rc = after_launch();
    prof_mark(p->prof_stop, s);
    return rc;
}

template <typename T, typename TO>
int generic_fwd_d(const Problem &P, const eagle_attn_params *p, cudaStream_t s) {
    switch (P.D) {
        case 32: return generic_fwd_launch<T, TO, 32>(P, p, s);
        case 64: return generic_fwd_launch<T, TO, 64>(P, p, s);
        case 128: return generic_fwd_launch<T, TO, 128>(P, p, s);
    }
    return EAGLE_ATTN_ERR_SHAPE;
}

int generic_fwd(const Problem &P, const eagle_attn_params *p, cudaStream_t s) {
    if (p->dtype == EAGLE_ATTN_F32) return generic_fwd_d<float, float>(P, p, s);
    if (p->out_dtype == EAGLE_ATTN_F32) return generic_fwd_d<__nv_bfloat16, float>(P, p, s);
    return generic_fwd_d<__nv_bfloat16, __nv_bfloat16>(P, p, s);
}

template <int D, typename TO>
int tc_fwd_run(const Problem &P, const eagle_attn_params *p, cudaStream_t s) {
    CUtensorMap tq, tk, tv;
    if (!make_q_tmap(&tq, p->q, P, tcfwd::BM) || !make_kv_tmap(&tk, p->cache_k, P, tcfwd::BN) ||
        !make_kv_tmap(&tv, p->cache_v, P, tcfwd::BN))
        return EAGLE_ATTN_ERR_CUDA;
    auto kern = tcfwd::fwd_kernel<D, TO>;
    const int smem = tcfwd::Cfg<D>::SMEM;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
        return EAGLE_ATTN_ERR_CUDA;
    dim3 grid(P.q_tiles ? (unsigned)p->num_q_tiles : (unsigned)((P.Tq + tcfwd::BM - 1) / tcfwd::BM),
              P.H, P.B);
    if (grid.x == 0) return EAGLE_ATTN_OK;
    prof_mark(p->prof_start, s);
    kern<<<grid, tcfwd::THREADS, smem, s>>>(tq, tk, tv, P, (TO *)p->out, p->lse);
    int rc = after_launch();
    prof_mark(p->prof_stop, s);
    return rc;
}

int tc_fwd_launch(const Problem &P, const eagle_attn_params *p, cudaStream_t s) {
    if (P.Tq == 0) return EAGLE_ATTN_OK;
    const bool f32out = p->out_dtype == EAGLE_ATTN_F32;
    if (P.D == 128)
        return f32out ? tc_fwd_run<128, float>(P, p, s) : tc_fwd_run<128, __nv_bfloat16>(P, p, s);
    if (P.D == 64)
        return f32out ? tc_fwd_run<64, float>(P, p, s) : tc_fwd_run<64, __nv_bfloat16>(P, p, s);
    return EAGLE_ATTN_ERR_UNSUPPORTED;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct BwdWorkspace {
    float *dq_acc;
    float *Dt;
};

size_t bwd_ws_bytes(const Problem &P) {
    return align256((size_t)P.B * P.Tq * P.H * P.D * 4) + align256((size_t)P.B * P.H * P.Tq * 4);
}

BwdWorkspace carve(const Problem &P, void *ws) {
    BwdWorkspace w;
    w.dq_acc = (float *)ws;
    w.Dt = (float *)((char *)ws + align256((size_t)P.B * P.Tq * P.H * P.D * 4));
    return w;
}

int64_t rows_of(const Problem &P) { return (int64_t)P.B * P.Tq * P.H; }

// dq = scale * dq_acc (fp32 [B, H, Tq, D]) in dq's dtype, or added to an fp32 dq.
template <int D>
int dq_finalize_launch(const Problem &P, const eagle_attn_params *p, const float *dq_acc,
                       cudaStream_t s) {
    constexpr int E = D / 32;
    const int64_t rows = row_slots(P);
    if (rows == 0) return EAGLE_ATTN_OK;
    dim3 grid((unsigned)((rows + 7) / 8));
    if (P.grad_accum)
        dq_finalize_kernel<float, E><<<grid, ROW_THREADS, 0, s>>>(P, dq_acc, (float *)p->dq);
    else
        dq_finalize_kernel<__nv_bfloat16, E><<<grid, ROW_THREADS, 0, s>>>(
            P, dq_acc, (__nv_bfloat16 *)p->dq);
    return after_launch();
}

template <int D>
int tc_bwd_run(const Problem &P, const eagle_attn_params *p, const float *Dws, float *dq_acc,
               bool has_diag, cudaStream_t s) {
    namespace kv = tcbwd::kv;
    namespace qk = tcbwd::qk;
    namespace kvq = tcbwd::kvq;
    static_assert(kv::BM == qk::BM && kv::BN == qk::BN && kv::BM == kv::BN &&
                      kvq::BM == kv::BM && kvq::BN == kv::BN,
                  "the backward kernels share one set of 128-row tensor maps");
    CUtensorMap tq, tdo, tk, tv;
    if (!make_q_tmap(&tq, p->q, P, kv::BM) || !make_q_tmap(&tdo, p->grad_out, P, kv::BM) ||
        !make_kv_tmap(&tk, p->cache_k, P, kv::BN) || !make_kv_tmap(&tv, p->cache_v, P, kv::BN))
        return EAGLE_ATTN_ERR_CUDA;
    if (!p->deterministic) {
        // one kernel, five products per tile pair; dQ summed in dq_acc (which the
        // row pass initialised), then scaled into dq
        // the accumulator [B, H, Tq, D] as rows x D, in the reduce-add boxes
        const int64_t acc_rows = (int64_t)P.B * P.H * P.Tq;
        if (acc_rows + kvq::BM > INT32_MAX) return EAGLE_ATTN_ERR_SHAPE;
        CUtensorMap tdq;
        if (!make_tmap_f32_2d(&tdq, dq_acc, (uint64_t)D, (uint64_t)acc_rows, kvq::DQ_BOX_COLS,
                              kvq::DQ_BOX_ROWS))
            return EAGLE_ATTN_ERR_CUDA;
        auto k = P.q_tiles ? kvq::dkdvdq_kernel<D, true> : kvq::dkdvdq_kernel<D, false>;
        const int sm = kvq::Cfg<D>::SMEM;
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) !=
            cudaSuccess)
            return EAGLE_ATTN_ERR_CUDA;
        prof_mark(p->prof_start, s);
        dim3 g((P.Tk + kvq::BN - 1) / kvq::BN, P.H, P.B);
        k<<<g, tcbwd::THREADS, sm, s>>>(tq, tdo, tk, tv, tdq, P, p->lse, Dws, p->dk, p->dv);
        if (after_launch()) return EAGLE_ATTN_ERR_CUDA;
        int rc = dq_finalize_launch<D>(P, p, dq_acc, s);
        prof_mark(p->prof_stop, s);
        return rc;
    }
    const float *dq_diag = has_diag ? dq_acc : nullptr;
    auto k1 = kv::dkdv_kernel<D>;
    auto k2 = qk::dq_kernel<D>;
    const int s1 = kv::Cfg<D>::SMEM, s2 = qk::Cfg<D>::SMEM;
    if (cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, s1) != cudaSuccess ||
        cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, s2) != cudaSuccess)
        return EAGLE_ATTN_ERR_CUDA;
    typedef __nv_bfloat16 bf;
    prof_mark(p->prof_start, s);
    dim3 g1((P.Tk + kv::BN - 1) / kv::BN, P.H, P.B);
    k1<<<g1, tcbwd::THREADS, s1, s>>>(tq, tdo, tk, tv, P, p->lse, Dws, p->dk, p->dv);
    if (after_launch()) return EAGLE_ATTN_ERR_CUDA;
    dim3 g2((P.Tq + qk::BM - 1) / qk::BM, P.H, P.B);
    k2<<<g2, tcbwd::THREADS, s2, s>>>(tq, tdo, tk, tv, P, p->lse, Dws, dq_diag, p->dq);
    int rc = after_launch();
    prof_mark(p->prof_stop, s);
    return rc;
}

int tc_bwd_launch(const Problem &P, const eagle_attn_params *p, const float *Dws, float *dq_acc,
                  bool has_diag, cudaStream_t s) {
    if (P.Tq == 0 && P.Tk == 0) return EAGLE_ATTN_OK;
    if (P.D == 128) return tc_bwd_run<128>(P, p, Dws, dq_acc, has_diag, s);
    if (P.D == 64) return tc_bwd_run<64>(P, p, Dws, dq_acc, has_diag, s);
    return EAGLE_ATTN_ERR_UNSUPPORTED;
}

template <typename T, typename TO, int E>
int bwd_prep_launch(const Problem &P, const eagle_attn_params *p, BwdWorkspace w, cudaStream_t s) {
    int64_t rows = rows_of(P);
    if (rows == 0) return EAGLE_ATTN_OK;
    dim3 grid((unsigned)((rows + 7) / 8));
    bwd_prep_kernel<T, TO, E><<<grid, ROW_THREADS, 0, s>>>(P, (const T *)p->grad_out,
                                                            (const TO *)p->out, w.Dt, w.dq_acc);
    return after_launch();
}

template <typename T, int E>
int bwd_diag_launch(const Problem &P, const eagle_attn_params *p, BwdWorkspace w, cudaStream_t s) {
    int64_t rows = rows_of(P);
    if (rows == 0) return EAGLE_ATTN_OK;
    dim3 grid((unsigned)((rows + 7) / 8));
    bwd_diag_kernel<T, E><<<grid, ROW_THREADS, 0, s>>>(
        P, (const T *)p->q, (const T *)p->cache_k, (const T *)p->cache_v, (const T *)p->grad_out,
        p->lse, w.Dt, w.dq_acc, (T *)p->dq, (T *)p->dk, (T *)p->dv);
    return after_launch();
}

template <typename T, int D>
int generic_bwd_main(const Problem &P, const eagle_attn_params *p, BwdWorkspace w,
                     cudaStream_t s) {
    const int smem = generic_bwd_smem_floats<D>() * 4;
    prof_mark(p->prof_start, s);
    if (P.Tk > 0) {
        auto k1 = generic_bwd_dkdv_kernel<T, D>;
        if (cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
            return EAGLE_ATTN_ERR_CUDA;
        dim3 g1((P.Tk + GT - 1) / GT, P.H, P.B);
        k1<<<g1, GTHREADS, smem, s>>>(P, (const T *)p->q, (const T *)p->cache_k,
                                       (const T *)p->cache_v, (const T *)p->grad_out, p->lse, w.Dt,
                                       (T *)p->dk, (T *)p->dv);
        if (after_launch()) return EAGLE_ATTN_ERR_CUDA;
    }
    if (P.Tq > 0 && P.Tk > 0) {
        auto k2 = generic_bwd_dq_kernel<T, D>;
        if (cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
            return EAGLE_ATTN_ERR_CUDA;
        dim3 g2((P.Tq + GT - 1) / GT, P.H, P.B);
        k2<<<g2, GTHREADS, smem, s>>>(P, (const T *)p->q, (const T *)p->cache_k,
                                       (const T *)p->cache_v, (const T *)p->grad_out, p->lse, w.Dt,
                                       w.dq_acc);
        if (after_launch()) return EAGLE_ATTN_ERR_CUDA;
    }
    prof_mark(p->prof_stop, s);
    return EAGLE_ATTN_OK;
}

template <typename T, typename TO, int D>
int bwd_all(const Problem &P, const eagle_attn_params *p, bool tc, cudaStream_t s) {
    constexpr int E = D / 32;
    BwdWorkspace w = carve(P, p->workspace);
    if (tc) {
        // tensor-core path: one row pass (D_t, diagonal grads, sum_i dz_i k_i
        // into the dQ workspace, zeros there without diagonal blocks when the
        // five-product kernel adds into it), then the block-0 kernels
        const int64_t rows = row_slots(P);
        const int zero_dq = p->deterministic ? 0 : 1;
        if (P.q_tiles && P.num_q_tiles > 0) {  // the list's order, on the device
            check_segments_kernel<<<1, 256, 0, s>>>(P);
            if (after_launch()) return EAGLE_ATTN_ERR_CUDA;
        }
        if (rows > 0) {
            dim3 grid((unsigned)((rows + 7) / 8));
            if (P.grad_accum)
                bwd_rows_kernel<T, TO, float, E><<<grid, ROW_THREADS, 0, s>>>(
                    P, (const T *)p->q, (const T *)p->cache_k, (const T *)p->cache_v,
                    (const T *)p->grad_out, (const TO *)p->out, p->lse, w.Dt, w.dq_acc,
                    (float *)p->dk, (float *)p->dv, zero_dq);
            else
                bwd_rows_kernel<T, TO, T, E><<<grid, ROW_THREADS, 0, s>>>(
                    P, (const T *)p->q, (const T *)p->cache_k, (const T *)p->cache_v,
                    (const T *)p->grad_out, (const TO *)p->out, p->lse, w.Dt, w.dq_acc,
                    (T *)p->dk, (T *)p->dv, zero_dq);
            if (after_launch()) return EAGLE_ATTN_ERR_CUDA;
        }
        return tc_bwd_launch(P, p, w.Dt, w.dq_acc, P.NB > 1, s);
    }
    int rc = bwd_prep_launch<T, TO, E>(P, p, w, s);
    if (rc) return rc;
    rc = generic_bwd_main<T, D>(P, p, w, s);
    if (rc) return rc;
    return bwd_diag_launch<T, E>(P, p, w, s);
}

template <typename T, typename TO>
int bwd_d(const Problem &P, const eagle_attn_params *p, bool tc, cudaStream_t s) {
    switch (P.D) {
        case 32: return bwd_all<T, TO, 32>(P, p, tc, s);
        case 64: return bwd_all<T, TO, 64>(P, p, tc, s);
        case 128: return bwd_all<T, TO, 128>(P, p, tc, s);
    }
    return EAGLE_ATTN_ERR_SHAPE;
}

}  // namespace

extern "C" {

int eagle_attn_abi_version(void) { return EAGLE_ATTN_ABI_VERSION; }

void eagle_attn_params_init(eagle_attn_params *p) {
    if (!p) return;
    memset(p, 0, sizeof(*p));
    p->struct_size = sizeof(eagle_attn_params);
    p->abi_version = EAGLE_ATTN_ABI_VERSION;
    p->dtype = EAGLE_ATTN_BF16;
    p->out_dtype = EAGLE_ATTN_BF16;
    p->impl = EAGLE_ATTN_IMPL_AUTO;
    p->causal = 1;
    p->scale = 1.0f;
}

int eagle_attn_fwd(const eagle_attn_params *p, void *stream) {
    Resolved r;
    int rc = resolve(p, false, &r);
    if (rc) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    rc = launch_check_cu(p, s);
    if (rc) return rc;
    if (r.tc) return tc_fwd_launch(r.P, p, s);
    return generic_fwd(r.P, p, s);
}

size_t eagle_attn_bwd_workspace_size(const eagle_attn_params *p) {
    if (!p || p->struct_size != sizeof(eagle_attn_params)) return 0;
    eagle_attn_params tmp = *p;
    // shapes only: pointers may still be unset
    const void *dummy = (const void *)(uintptr_t)256;
    tmp.q = tmp.cache_k = tmp.cache_v = tmp.grad_out = dummy;
    tmp.out = tmp.dq = tmp.dk = tmp.dv = (void *)dummy;
    tmp.lse = (float *)dummy;
    tmp.workspace = nullptr;
    Resolved r;
    if (resolve(&tmp, true, &r)) return 0;
    return bwd_ws_bytes(r.P);
}

int eagle_attn_bwd(const eagle_attn_params *p, void *stream) {
    Resolved r;
    int rc = resolve(p, true, &r);
    if (rc) return rc;
    if (!p->workspace || p->workspace_bytes < bwd_ws_bytes(r.P)) return EAGLE_ATTN_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    rc = launch_check_cu(p, s);
    if (rc) return rc;
    const Problem &P = r.P;
    if (p->dtype == EAGLE_ATTN_F32) return bwd_d<float, float>(P, p, r.tc, s);
    if (p->out_dtype == EAGLE_ATTN_F32) return bwd_d<__nv_bfloat16, float>(P, p, r.tc, s);
    return bwd_d<__nv_bfloat16, __nv_bfloat16>(P, p, r.tc, s);
}

int attn_merge_out_lse(float *out, float *lse, const void *block_out, int block_dtype,
                       const float *block_lse, int B, int T, int H, int D, int init,
                       void *stream) {
    if (!out || !lse || !block_out || !block_lse) return EAGLE_ATTN_ERR_NULL;
    if (block_dtype != EAGLE_ATTN_F32 && block_dtype != EAGLE_ATTN_BF16) return EAGLE_ATTN_ERR_DTYPE;
    if (B < 1 || T < 0 || H < 1 || (D != 64 && D != 128) || H > 65535 || B > 65535)
        return EAGLE_ATTN_ERR_SHAPE;
    if (!aligned16(out) || !aligned16(block_out) || ((uintptr_t)lse & 3) || ((uintptr_t)block_lse & 3))
        return EAGLE_ATTN_ERR_ALIGN;
    if (block_dtype == EAGLE_ATTN_BF16 && D % 8 && ((uintptr_t)block_out & 7))
        return EAGLE_ATTN_ERR_ALIGN;
    if ((int64_t)B * T * H == 0) return EAGLE_ATTN_OK;
    if (D != 64 && D != 128) return EAGLE_ATTN_ERR_SHAPE;
    cudaStream_t s = (cudaStream_t)stream;
    const int tpb = (MERGE_THREADS / 32) * MERGE_TW;
    if ((T + tpb - 1) / tpb > 65535) return EAGLE_ATTN_ERR_SHAPE;
    dim3 grid((unsigned)H, (unsigned)((T + tpb - 1) / tpb), (unsigned)B);
#define EAGLE_MERGE(TB, D4)                                                                  \
    merge_kernel<TB, D4><<<grid, MERGE_THREADS, 0, s>>>(out, lse, (const TB *)block_out,      \
                                                        block_lse, T, H, init)
    if (block_dtype == EAGLE_ATTN_F32) {
        if (D == 128) EAGLE_MERGE(float, 32); else EAGLE_MERGE(float, 16);
    } else {
        if (D == 128) EAGLE_MERGE(__nv_bfloat16, 32); else EAGLE_MERGE(__nv_bfloat16, 16);
    }
#undef EAGLE_MERGE
    return after_launch();
}

int attn_merge_diag(const eagle_attn_params *p, void *stream) {
    if (!p) return EAGLE_ATTN_ERR_NULL;
    eagle_attn_params tmp = *p;
    if (tmp.out_dtype != EAGLE_ATTN_F32) return EAGLE_ATTN_ERR_DTYPE;
    tmp.impl = EAGLE_ATTN_IMPL_GENERIC;
    tmp.cu_seqlens = nullptr;
    tmp.q_tiles = nullptr;  // every row of the running state
    tmp.q_tile_rows = nullptr;
    Resolved r;
    int rc = resolve(&tmp, false, &r);
    if (rc) return rc;
    if (p->num_blocks < 2) return EAGLE_ATTN_OK;
    const Problem &P = r.P;
    int64_t rows = rows_of(P);
    if (rows == 0) return EAGLE_ATTN_OK;
    cudaStream_t s = (cudaStream_t)stream;
    dim3 grid((unsigned)((rows + 7) / 8));
#define EAGLE_DIAG(T, E)                                                                      \
    merge_diag_kernel<T, E><<<grid, ROW_THREADS, 0, s>>>(P, (const T *)p->q,                 \
                                                         (const T *)p->cache_k,              \
                                                         (const T *)p->cache_v, (float *)p->out, \
                                                         p->lse)
    if (p->dtype == EAGLE_ATTN_F32) {
        if (P.D == 32) EAGLE_DIAG(float, 1);
        else if (P.D == 64) EAGLE_DIAG(float, 2);
        else EAGLE_DIAG(float, 4);
    } else {
        if (P.D == 32) EAGLE_DIAG(__nv_bfloat16, 1);
        else if (P.D == 64) EAGLE_DIAG(__nv_bfloat16, 2);
        else EAGLE_DIAG(__nv_bfloat16, 4);
    }
#undef EAGLE_DIAG
    return after_launch();
}

int attn_finalize(const float *src, void *dst, int dst_dtype, size_t count, void *stream) {
    if (!src || !dst) return EAGLE_ATTN_ERR_NULL;
    if (dst_dtype != EAGLE_ATTN_F32 && dst_dtype != EAGLE_ATTN_BF16) return EAGLE_ATTN_ERR_DTYPE;
    const uintptr_t dst_align = dst_dtype == EAGLE_ATTN_F32 ? 4 : 2;
    if (((uintptr_t)src & 3) || ((uintptr_t)dst & (dst_align - 1))) return EAGLE_ATTN_ERR_ALIGN;
    if (count == 0) return EAGLE_ATTN_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (!aligned16(src) || !aligned16(dst)) {
        dim3 grid((unsigned)((count + 255) / 256));
        if (dst_dtype == EAGLE_ATTN_F32)
            finalize_scalar_kernel<float><<<grid, 256, 0, s>>>(src, (float *)dst, count);
        else
            finalize_scalar_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(src, (__nv_bfloat16 *)dst,
                                                                       count);
        return after_launch();
    }
    size_t threads = (count + 3) / 4;
    dim3 grid((unsigned)((threads + 255) / 256));
    if (dst_dtype == EAGLE_ATTN_F32)
        finalize_kernel<float><<<grid, 256, 0, s>>>(src, (float *)dst, count);
    else
        finalize_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(src, (__nv_bfloat16 *)dst, count);
    return after_launch();
}

int eagle_attn_get_status(int *code) {
    if (!code) return EAGLE_ATTN_ERR_NULL;
    return cuda_status(cudaMemcpyFromSymbol(code, g_status, sizeof(int)));
}

int eagle_attn_clear_status(void) {
    int zero = 0;
    return cuda_status(cudaMemcpyToSymbol(g_status, &zero, sizeof(int)));
}

}  // extern "C"

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current) and cached.
int noalloc_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return EAGLE_ATTN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return EAGLE_ATTN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
            return EAGLE_ATTN_ERR_CUDA;
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return EAGLE_ATTN_OK;
}

}  // namespace

extern "C" {

int eagle_attn_bwd_noalloc(const eagle_attn_params *p, void *stream) {
    if (!p) return EAGLE_ATTN_ERR_NULL;
    // the caller's workspace fields are ignored: validate without them
    eagle_attn_params q = *p;
    q.workspace = nullptr;
    q.workspace_bytes = 0;
    Resolved r;
    int rc = resolve(&q, true, &r);
    if (rc) return rc;
    if (bwd_ws_bytes(r.P) > (size_t)EAGLE_ATTN_NOALLOC_SCRATCH_BYTES)
        return EAGLE_ATTN_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc) return rc;
    q.workspace = scratch;
    q.workspace_bytes = EAGLE_ATTN_NOALLOC_SCRATCH_BYTES;
    return eagle_attn_bwd(&q, stream);
}

int eagle_attn_selftest_wait_timeout(int64_t limit_ns, void *stream) {
    if (limit_ns < 1 || limit_ns > 1000000000) return EAGLE_ATTN_ERR_SHAPE;
    wait_timeout_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_ns);
    return after_launch();
}

uint64_t eagle_attn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *eagle_attn_strerror(int code) {
    switch (code) {
        case EAGLE_ATTN_OK: return "ok";
        case EAGLE_ATTN_ERR_NULL: return "a required pointer is NULL";
        case EAGLE_ATTN_ERR_ABI: return "abi_version or struct_size mismatch";
        case EAGLE_ATTN_ERR_DTYPE: return "unsupported dtype";
        case EAGLE_ATTN_ERR_SHAPE: return "bad shape";
        case EAGLE_ATTN_ERR_STRIDE: return "bad strides";
        case EAGLE_ATTN_ERR_ALIGN: return "pointer or stride not 16-byte aligned";
        case EAGLE_ATTN_ERR_VARLEN: return "cu_seqlens requires B == 1 and num_docs >= 1";
        case EAGLE_ATTN_ERR_WORKSPACE: return "workspace missing or too small";
        case EAGLE_ATTN_ERR_UNSUPPORTED: return "no kernel serves this request";
        case EAGLE_ATTN_ERR_CUDA: return "CUDA runtime error";
        case EAGLE_ATTN_ERR_DEVICE: return "device-side check failed";
        case EAGLE_ATTN_ERR_SCRATCH_LIMIT:
            return "problem needs more scratch than the no-allocation backward's fixed buffer holds";
    }
    return "unknown status";
}

}  // extern "C"
