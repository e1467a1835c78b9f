// sa3.cu -- libsa3: the C ABI declared in include/sa3.h.
//
// Single translation unit: the quantizer (quant.cuh) and attention kernel
// (attn.cuh) are included here so that the device status word below is one
// object without relocatable device code.  Host code validates arguments,
// encodes the TMA tensor maps and enqueues the kernels on the caller's
// stream; it allocates nothing.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "sa3.h"

// Only the C entry points of sa3.h are exported.  The kernels, their host
// stubs and launchers stay hidden, so that a second build of this library
// (or any library with the same template instances) loaded into the process
// can neither bind to them nor interpose its own.
#pragma GCC visibility push(hidden)
#include "sa3_internal.h"
#include "sm100.cuh"

#include "attn.cuh"
#include "attn8.cuh"
#include "probe.cuh"
#include "quant.cuh"
#pragma GCC visibility pop

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 2-D byte tensor [rows][inner] with a box of box_rows x box_inner bytes.
bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint32_t box_inner,
              uint32_t box_rows, CUtensorMapSwizzle sw) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [BH][N][d] as a 3-D tensor {d, N, BH}: boxes of 64 channels x 128
// tokens x 1 head, 128-byte swizzle; tokens past N read as zeros.
bool make_qkv_map(CUtensorMap *m, const void *base, int d, int N, int BH) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
    const cuuint32_t box[3] = {64, 128, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Byte range [p, p + n) of a buffer.
struct Range {
    uintptr_t lo, hi;
};
Range range_of(const void *p, int64_t n) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Range{a, a + static_cast<uintptr_t>(n)};
}
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

// True if any written range overlaps any input range.  Every launch here
// has CTAs reading inputs while others write outputs (the quantizer's
// second launch also loads K before it waits for the first), so an output
// that aliases an input would race with those reads.
bool any_overlap(const Range *in, int nin, const Range *out, int nout) {
    for (int i = 0; i < nin; ++i)
        for (int o = 0; o < nout; ++o)
            if (overlap(in[i], out[o])) return true;
    return false;
}
bool aligned32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

int check_shape(int B, int H, int N, int d) {
    if (B < 1 || H < 1 || N < 1) return SA3_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SA3_ERR_UNSUPPORTED;
    const int64_t BH = static_cast<int64_t>(B) * H;
    const int64_t Np = sa3_padded_len(N);
    if (BH * Np * d / 2 >= (int64_t(1) << 31) || BH * Np >= (int64_t(1) << 31)) return SA3_ERR_UNSUPPORTED;
    return SA3_OK;
}

// need_q: the Q code and scale buffers are used (not so when Q is skipped
// by the quantizer or quantized on load by the attention kernel).
int check_qkv(const sa3_qkv_fp4 *t, bool need_q = true) {
    if (!t || (need_q && (!t->q_fp4 || !t->q_sf)) || !t->k_fp4 || !t->k_sf || !t->vt_fp4 || !t->vt_sf || !t->k_mean)
        return SA3_ERR_INVALID_ARG;
    if ((need_q && (!aligned16(t->q_fp4) || !aligned16(t->q_sf))) || !aligned16(t->k_fp4) || !aligned16(t->k_sf) ||
        !aligned16(t->vt_fp4) || !aligned16(t->vt_sf) || !aligned16(t->k_mean))
        return SA3_ERR_INVALID_ARG;
    return SA3_OK;
}

// Self-test of the bounded waits: one warp waits on an mbarrier that nothing
// ever arrives on, through the same routine the attention kernel uses, so
// the wait must give up after `limit_ns` and record the timeout.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sa3::mbar_init(&bar, 1);
        abort_flag = 0;
        sa3::fence_mbar_init();
    }
    __syncwarp();
    sa3::mbar_wait_limit(&bar, 0, &abort_flag, limit_ns);
}

// Scratch for sa3_quantize_qkv_noalloc: one fixed array per device that
// loads the library (fp64 K-mean partial sums).
static __device__ __align__(256) double g_noalloc_scratch[SA3_NOALLOC_SCRATCH_BYTES / sizeof(double)];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of this device's scratch array, looked up once per device
// with that device current (host code must not pass the symbol itself).
void *noalloc_scratch(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = ptr;
    }
    return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" {

const char *sa3_version(void) { return "libsa3 0.1.0 (sm_100a)"; }

int sa3_quantize_qkv_ex(const void *q, const void *k, const void *v, int B, int H, int Nq, int Nkv, int d,
                        unsigned int flags, const sa3_qkv_fp4 *out, float *v_mean, void *workspace,
                        size_t workspace_bytes, struct CUstream_st *stream) {
    int rc = check_shape(B, H, Nq, d);
    if (rc != SA3_OK || (rc = check_shape(B, H, Nkv, d)) != SA3_OK) return rc;
    if ((flags & ~static_cast<unsigned int>(SA3_V_SMOOTH | SA3_SKIP_Q)) != 0) return SA3_ERR_INVALID_ARG;
    const bool vsmooth = (flags & SA3_V_SMOOTH) != 0;
    const bool skip_q = (flags & SA3_SKIP_Q) != 0;
    if ((!skip_q && (!q || !aligned16(q))) || !k || !v || !aligned16(k) || !aligned16(v)) return SA3_ERR_INVALID_ARG;
    if ((rc = check_qkv(out, !skip_q)) != SA3_OK) return rc;
    if (vsmooth && (!v_mean || !aligned16(v_mean))) return SA3_ERR_INVALID_ARG;
    const int64_t need = sa3_quant_workspace_bytes_ex(B, H, Nkv, d, flags);
    if (!workspace || !aligned16(workspace) || workspace_bytes < static_cast<size_t>(need)) return SA3_ERR_INVALID_ARG;
    {
        const Range in[3] = {range_of(skip_q ? nullptr : q, skip_q ? 0 : int64_t(B) * H * Nq * d * 2),
                             range_of(k, int64_t(B) * H * Nkv * d * 2), range_of(v, int64_t(B) * H * Nkv * d * 2)};
        const Range wr[9] = {range_of(out->q_fp4, skip_q ? 0 : sa3_qk_fp4_bytes(B, H, Nq, d)),
                             range_of(out->q_sf, skip_q ? 0 : sa3_qk_sf_bytes(B, H, Nq, d)),
                             range_of(out->k_fp4, sa3_qk_fp4_bytes(B, H, Nkv, d)),
                             range_of(out->k_sf, sa3_qk_sf_bytes(B, H, Nkv, d)),
                             range_of(out->vt_fp4, sa3_vt_fp4_bytes(B, H, Nkv, d)),
                             range_of(out->vt_sf, sa3_vt_sf_bytes(B, H, Nkv, d)),
                             range_of(out->k_mean, sa3_kmean_bytes(B, H, d)), range_of(workspace, need),
                             range_of(v_mean, vsmooth ? sa3_kmean_bytes(B, H, d) : 0)};
        if (any_overlap(in, 3, wr, 9)) return SA3_ERR_INVALID_ARG;
    }
    sa3::QuantParams p = {};
    p.q_fp4 = static_cast<uint8_t *>(out->q_fp4);
    p.q_sf = static_cast<uint8_t *>(out->q_sf);
    p.k_fp4 = static_cast<uint8_t *>(out->k_fp4);
    p.k_sf = static_cast<uint8_t *>(out->k_sf);
    p.vt_fp4 = static_cast<uint8_t *>(out->vt_fp4);
    p.vt_sf = static_cast<uint8_t *>(out->vt_sf);
    p.k_mean = out->k_mean;
    p.part = static_cast<double *>(workspace);
    p.BH = B * H;
    p.N = Nkv;
    p.Np = static_cast<int>(sa3_padded_len(Nkv));
    // skipping Q: a schedule without Q tiles
    p.Nq = skip_q ? 0 : Nq;
    p.Npq = skip_q ? 0 : static_cast<int>(sa3_padded_len(Nq));
    p.chunk = static_cast<int>(sa3_kmean_chunk(Nkv));
    p.nchunk = static_cast<int>(sa3_kmean_nchunk(Nkv));
    p.st32 = (skip_q || aligned32(p.q_fp4)) && aligned32(p.k_fp4);
    p.vsmooth = vsmooth ? 1 : 0;
    p.v_mean = v_mean;
    p.vpart = p.part + static_cast<size_t>(p.BH) * p.nchunk * d;
    CUtensorMap tq, tk, tv;
    if (!make_qkv_map(&tk, k, d, Nkv, p.BH) || !make_qkv_map(&tv, v, d, Nkv, p.BH) ||
        !(skip_q ? make_qkv_map(&tq, k, d, Nkv, p.BH) : make_qkv_map(&tq, q, d, Nq, p.BH)))
        return SA3_ERR_CUDA;
    return sa3::launch_quant(p, tq, tk, tv, d, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? SA3_OK
                                                                                                        : SA3_ERR_CUDA;
}

int sa3_quantize_qkv_lens(const void *q, const void *k, const void *v, int B, int H, int Nq, int Nkv, int d,
                          const sa3_qkv_fp4 *out, void *workspace, size_t workspace_bytes,
                          struct CUstream_st *stream) {
    return sa3_quantize_qkv_ex(q, k, v, B, H, Nq, Nkv, d, 0u, out, nullptr, workspace, workspace_bytes, stream);
}

int sa3_quantize_qkv_i8(const void *q, const void *k, const void *v, int B, int H, int Nq, int Nkv, int d,
                        const sa3_qkv_i8 *out, void *workspace, size_t workspace_bytes,
                        struct CUstream_st *stream) {
    int rc = check_shape(B, H, Nq, d);
    if (rc != SA3_OK || (rc = check_shape(B, H, Nkv, d)) != SA3_OK) return rc;
    if (!q || !k || !v || !aligned16(q) || !aligned16(k) || !aligned16(v)) return SA3_ERR_INVALID_ARG;
    if (!out || !out->q_i8 || !out->q_scale || !out->k_i8 || !out->k_scale || !out->vt_f16 || !out->k_mean ||
        !aligned16(out->q_i8) || !aligned16(out->q_scale) || !aligned16(out->k_i8) || !aligned16(out->k_scale) ||
        !aligned16(out->vt_f16) || !aligned16(out->k_mean))
        return SA3_ERR_INVALID_ARG;
    const int64_t need = sa3_quant_workspace_bytes(B, H, Nkv, d);
    if (!workspace || !aligned16(workspace) || workspace_bytes < static_cast<size_t>(need)) return SA3_ERR_INVALID_ARG;
    {
        const Range in[3] = {range_of(q, int64_t(B) * H * Nq * d * 2), range_of(k, int64_t(B) * H * Nkv * d * 2),
                             range_of(v, int64_t(B) * H * Nkv * d * 2)};
        const Range wr[7] = {range_of(out->q_i8, sa3_i8_bytes(B, H, Nq, d)),
                             range_of(out->q_scale, sa3_i8_scale_bytes(B, H, Nq)),
                             range_of(out->k_i8, sa3_i8_bytes(B, H, Nkv, d)),
                             range_of(out->k_scale, sa3_i8_scale_bytes(B, H, Nkv)),
                             range_of(out->vt_f16, sa3_vt_f16_bytes(B, H, Nkv, d)),
                             range_of(out->k_mean, sa3_kmean_bytes(B, H, d)), range_of(workspace, need)};
        if (any_overlap(in, 3, wr, 7)) return SA3_ERR_INVALID_ARG;
    }
    sa3::QuantParams p = {};
    p.q_fp4 = static_cast<uint8_t *>(out->q_i8);
    p.k_fp4 = static_cast<uint8_t *>(out->k_i8);
    p.vt_fp4 = static_cast<uint8_t *>(out->vt_f16);
    p.q_scale = out->q_scale;
    p.k_scale = out->k_scale;
    p.k_mean = out->k_mean;
    p.part = static_cast<double *>(workspace);
    p.BH = B * H;
    p.N = Nkv;
    p.Np = static_cast<int>(sa3_padded_len(Nkv));
    p.Nq = Nq;
    p.Npq = static_cast<int>(sa3_padded_len(Nq));
    p.chunk = static_cast<int>(sa3_kmean_chunk(Nkv));
    p.nchunk = static_cast<int>(sa3_kmean_nchunk(Nkv));
    p.st32 = aligned32(p.q_fp4) && aligned32(p.k_fp4) && aligned32(p.vt_fp4);
    CUtensorMap tq, tk, tv;
    if (!make_qkv_map(&tq, q, d, Nq, p.BH) || !make_qkv_map(&tk, k, d, Nkv, p.BH) ||
        !make_qkv_map(&tv, v, d, Nkv, p.BH))
        return SA3_ERR_CUDA;
    return sa3::launch_quant_i8(p, tq, tk, tv, d, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SA3_OK
               : SA3_ERR_CUDA;
}

int sa3_quantize_qkv(const void *q, const void *k, const void *v, int B, int H, int N, int d,
                     const sa3_qkv_fp4 *out, void *workspace, size_t workspace_bytes, struct CUstream_st *stream) {
    return sa3_quantize_qkv_lens(q, k, v, B, H, N, N, d, out, workspace, workspace_bytes, stream);
}

int sa3_quantize_qkv_noalloc(const void *q, const void *k, const void *v, int B, int H, int N, int d,
                             const sa3_qkv_fp4 *out, struct CUstream_st *stream) {
    int rc = check_shape(B, H, N, d);
    if (rc != SA3_OK) return rc;
    if (!q || !k || !v || !aligned16(q) || !aligned16(k) || !aligned16(v)) return SA3_ERR_INVALID_ARG;
    if ((rc = check_qkv(out)) != SA3_OK) return rc;
    if (sa3_quant_workspace_bytes(B, H, N, d) > static_cast<int64_t>(SA3_NOALLOC_SCRATCH_BYTES))
        return SA3_ERR_UNSUPPORTED;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return SA3_ERR_CUDA;
    void *scratch = noalloc_scratch(dev);
    if (!scratch) return SA3_ERR_CUDA;
    return sa3_quantize_qkv(q, k, v, B, H, N, d, out, scratch, SA3_NOALLOC_SCRATCH_BYTES, stream);
}

int sa3_attn_fwd_ex(const sa3_qkv_fp4 *in, const void *q, const float *v_mean, int B, int H, int Nq, int Nkv,
                    int d, int causal, float sm_scale, unsigned int flags, void *out, struct CUstream_st *stream) {
    int rc = check_shape(B, H, Nq, d);
    if (rc != SA3_OK || (rc = check_shape(B, H, Nkv, d)) != SA3_OK) return rc;
    if ((flags & ~static_cast<unsigned int>(SA3_P_TWO_LEVEL | SA3_V_SMOOTH | SA3_Q_ON_LOAD)) != 0)
        return SA3_ERR_INVALID_ARG;
    const bool q_load = (flags & SA3_Q_ON_LOAD) != 0;
    if ((rc = check_qkv(in, !q_load)) != SA3_OK) return rc;
    if (q_load && (!q || !aligned16(q))) return SA3_ERR_INVALID_ARG;
    if (!out || !aligned16(out) || (causal != 0 && causal != 1)) return SA3_ERR_INVALID_ARG;
    if ((flags & SA3_V_SMOOTH) && (!v_mean || !aligned16(v_mean))) return SA3_ERR_INVALID_ARG;
    {
        // the output must not share bytes with any input: other CTAs may
        // still be reading an input (Q on load above all) while one writes
        const Range wr[1] = {range_of(out, int64_t(B) * H * Nq * d * 2)};
        const Range rd[8] = {range_of(q_load ? nullptr : in->q_fp4, q_load ? 0 : sa3_qk_fp4_bytes(B, H, Nq, d)),
                             range_of(q_load ? nullptr : in->q_sf, q_load ? 0 : sa3_qk_sf_bytes(B, H, Nq, d)),
                             range_of(in->k_fp4, sa3_qk_fp4_bytes(B, H, Nkv, d)),
                             range_of(in->k_sf, sa3_qk_sf_bytes(B, H, Nkv, d)),
                             range_of(in->vt_fp4, sa3_vt_fp4_bytes(B, H, Nkv, d)),
                             range_of(in->vt_sf, sa3_vt_sf_bytes(B, H, Nkv, d)),
                             range_of(q_load ? q : nullptr, q_load ? int64_t(B) * H * Nq * d * 2 : 0),
                             range_of((flags & SA3_V_SMOOTH) ? v_mean : nullptr,
                                      (flags & SA3_V_SMOOTH) ? sa3_kmean_bytes(B, H, d) : 0)};
        if (any_overlap(rd, 8, wr, 1)) return SA3_ERR_INVALID_ARG;
    }
    if (!(sm_scale > 0.0f)) sm_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
    if (!std::isfinite(sm_scale)) return SA3_ERR_INVALID_ARG;
    const int BH = B * H;
    const int Npq = static_cast<int>(sa3_padded_len(Nq));
    const int Np = static_cast<int>(sa3_padded_len(Nkv));
    CUtensorMap tq, tk, tv;
    const CUtensorMapSwizzle qk_sw = d == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
    if (!(q_load ? make_qkv_map(&tq, q, d, Nq, BH)
                 : make_map(&tq, in->q_fp4, d / 2, static_cast<uint64_t>(BH) * Npq, d / 2, 128, qk_sw)) ||
        !make_map(&tk, in->k_fp4, d / 2, static_cast<uint64_t>(BH) * Np, d / 2, 128, qk_sw) ||
        !make_map(&tv, in->vt_fp4, Np / 2, static_cast<uint64_t>(BH) * d, 64, d, CU_TENSOR_MAP_SWIZZLE_64B))
        return SA3_ERR_CUDA;
    sa3::AttnParams p = {};
    p.q_sf = static_cast<const uint8_t *>(in->q_sf);
    p.k_sf = static_cast<const uint8_t *>(in->k_sf);
    p.vt_sf = static_cast<const uint8_t *>(in->vt_sf);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.v_mean = (flags & SA3_V_SMOOTH) ? v_mean : nullptr;
    p.q_load = q_load ? 1 : 0;
    p.BH = BH;
    p.N = Nkv;
    p.Np = Np;
    p.Nq = Nq;
    p.Npq = Npq;
    p.causal = causal;
    p.scale_log2 = static_cast<float>(static_cast<double>(sm_scale) * 1.4426950408889634);
    p.p_pre_log2 = (flags & SA3_P_TWO_LEVEL) ? 11.0f : 0.0f;
    return sa3::launch_attn(p, tq, tk, tv, d, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SA3_OK
               : SA3_ERR_CUDA;
}

int sa3_attn_fwd_lens(const sa3_qkv_fp4 *in, int B, int H, int Nq, int Nkv, int d, int causal, float sm_scale,
                      unsigned int flags, void *out, struct CUstream_st *stream) {
    if ((flags & ~static_cast<unsigned int>(SA3_P_TWO_LEVEL)) != 0) return SA3_ERR_INVALID_ARG;
    return sa3_attn_fwd_ex(in, nullptr, nullptr, B, H, Nq, Nkv, d, causal, sm_scale, flags, out, stream);
}

int sa3_attn_fwd_i8_lse(const sa3_qkv_i8 *in, int B, int H, int Nq, int Nkv, int d, int causal, float sm_scale,
                        void *out, float *lse, struct CUstream_st *stream) {
    int rc = check_shape(B, H, Nq, d);
    if (rc != SA3_OK || (rc = check_shape(B, H, Nkv, d)) != SA3_OK) return rc;
    if (!in || !in->q_i8 || !in->q_scale || !in->k_i8 || !in->k_scale || !in->vt_f16 || !aligned16(in->q_i8) ||
        !aligned16(in->k_i8) || !aligned16(in->vt_f16))
        return SA3_ERR_INVALID_ARG;
    if (!out || !aligned16(out) || (causal != 0 && causal != 1)) return SA3_ERR_INVALID_ARG;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return SA3_ERR_INVALID_ARG;
    {
        // no output may share bytes with an input or with the other output
        const Range wr[2] = {range_of(out, int64_t(B) * H * Nq * d * 2),
                             range_of(lse, lse ? int64_t(B) * H * Nq * 4 : 0)};
        const Range rd[5] = {range_of(in->q_i8, sa3_i8_bytes(B, H, Nq, d)),
                             range_of(in->q_scale, sa3_i8_scale_bytes(B, H, Nq)),
                             range_of(in->k_i8, sa3_i8_bytes(B, H, Nkv, d)),
                             range_of(in->k_scale, sa3_i8_scale_bytes(B, H, Nkv)),
                             range_of(in->vt_f16, sa3_vt_f16_bytes(B, H, Nkv, d))};
        if (any_overlap(rd, 5, wr, 2) || overlap(wr[0], wr[1])) return SA3_ERR_INVALID_ARG;
    }
    if (!(sm_scale > 0.0f)) sm_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
    if (!std::isfinite(sm_scale)) return SA3_ERR_INVALID_ARG;
    const int BH = B * H;
    const int Npq = static_cast<int>(sa3_padded_len(Nq));
    const int Np = static_cast<int>(sa3_padded_len(Nkv));
    CUtensorMap tq, tk, tv;
    const CUtensorMapSwizzle qk_sw = d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    if (!make_map(&tq, in->q_i8, d, static_cast<uint64_t>(BH) * Npq, d, 128, qk_sw) ||
        !make_map(&tk, in->k_i8, d, static_cast<uint64_t>(BH) * Np, d, 128, qk_sw) ||
        !make_map(&tv, in->vt_f16, static_cast<uint64_t>(Np) * 2, static_cast<uint64_t>(BH) * d, 128, d,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return SA3_ERR_CUDA;
    sa3::AttnParams p = {};
    p.q_scale = in->q_scale;
    p.k_scale = in->k_scale;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.BH = BH;
    p.N = Nkv;
    p.Np = Np;
    p.Nq = Nq;
    p.Npq = Npq;
    p.causal = causal;
    p.scale_log2 = static_cast<float>(static_cast<double>(sm_scale) * 1.4426950408889634);
    return sa3::launch_attn_i8(p, tq, tk, tv, d, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SA3_OK
               : SA3_ERR_CUDA;
}

int sa3_attn_fwd_i8(const sa3_qkv_i8 *in, int B, int H, int Nq, int Nkv, int d, int causal, float sm_scale,
                    void *out, struct CUstream_st *stream) {
    return sa3_attn_fwd_i8_lse(in, B, H, Nq, Nkv, d, causal, sm_scale, out, nullptr, stream);
}

int sa3_attn_fwd(const sa3_qkv_fp4 *in, int B, int H, int N, int d, int causal, float sm_scale, void *out,
                 struct CUstream_st *stream) {
    return sa3_attn_fwd_lens(in, B, H, N, N, d, causal, sm_scale, 0u, out, stream);
}

int sa3_probe_fp4_mma(int ctas, int n, int iters, float *out, struct CUstream_st *stream) {
    if (ctas < 1 || ctas > 65535 || iters < 1 || iters > (1 << 18) || !out || (n != 128 && n != 256) ||
        (reinterpret_cast<uintptr_t>(out) & 3u))
        return SA3_ERR_INVALID_ARG;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e = n == 128 ? sa3::probe::launch<128>(ctas, iters, out, s)
                                   : sa3::probe::launch<256>(ctas, iters, out, s);
    return e == cudaSuccess ? SA3_OK : SA3_ERR_CUDA;
}

int sa3_selftest_wait_timeout(unsigned int limit_us, struct CUstream_st *stream) {
    if (limit_us == 0 || limit_us > 10u * 1000u * 1000u) return SA3_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<uint64_t>(limit_us) * 1000ull);
    return cudaGetLastError() == cudaSuccess ? SA3_OK : SA3_ERR_CUDA;
}

int sa3_device_status(struct CUstream_st *stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return SA3_ERR_CUDA;
    unsigned int st = 0;
    if (cudaMemcpyFromSymbol(&st, sa3::g_sa3_status, sizeof(st)) != cudaSuccess) return SA3_ERR_CUDA;
    if (st != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(sa3::g_sa3_status, &zero, sizeof(zero)) != cudaSuccess) return SA3_ERR_CUDA;
        return SA3_ERR_TIMEOUT;
    }
    return SA3_OK;
}

}  // extern "C"
