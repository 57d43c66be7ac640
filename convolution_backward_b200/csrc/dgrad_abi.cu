// dgrad_abi.cu -- the C ABI of libdgrad (declared in include/dgrad.h).
//
// Host side only: argument validation (everything is checked before anything
// is launched), TMA tensor-map encoding for the tensor-core kernel, the per-device
// status word the kernels report timeouts into, and dispatch to the kernels.
// Also two diagnostics: a self-test kernel whose bounded wait is made to run
// out (it checks the timeout path without hanging anything) and an FMA-rate
// probe used to measure the fp32 roofline.
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "dgrad.h"
#include "host_util.h"
#include "launchers.h"

namespace {

thread_local int t_last_cuda = 0;

// One status word per device: module-scope device variables exist once per
// device context that loads the library.
__device__ int g_status_word;

struct DeviceState {
    bool ready = false;
    int* status = nullptr;   // device address of g_status_word on that device
    int sms = 0;
};

constexpr int kMaxDevices = 64;
DeviceState g_devices[kMaxDevices];
std::mutex g_mu;

dgrad_status_t cuda_fail(cudaError_t e)
{
    t_last_cuda = static_cast<int>(e);
    return DGRAD_ERR_CUDA;
}

dgrad_status_t device_state(DeviceState** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return DGRAD_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState& st = g_devices[dev];
    if (!st.ready) {
        void* addr = nullptr;
        e = cudaGetSymbolAddress(&addr, g_status_word);
        if (e != cudaSuccess) return cuda_fail(e);
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e);
        st.status = static_cast<int*>(addr);
        st.sms = sms;
        st.ready = true;
    }
    *out = &st;
    return DGRAD_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Encoded tensor maps, kept per (type, base, extents, strides, box, swizzle):
// a caller that repeats a call on the same buffers (the common case) reuses the
// map instead of encoding it again.  A small table with round-robin replacement.
struct MapKey {
    int dtype, rank, swizzle, promo;
    const void* base;
    cuuint64_t dims[5], strides[4];
    cuuint32_t box[5];
    bool operator==(const MapKey& o) const { return memcmp(this, &o, sizeof(MapKey)) == 0; }
};

CUresult encode_cached(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, CUtensorMapDataType dtype,
                       cuuint32_t rank, void* base, const cuuint64_t* dims, const cuuint64_t* strides,
                       const cuuint32_t* box, const cuuint32_t* estr, CUtensorMapSwizzle swz,
                       CUtensorMapL2promotion promo)
{
    constexpr int kSlots = 128;
    static MapKey keys[kSlots];
    static CUtensorMap maps[kSlots];
    static bool used[kSlots];
    static int next = 0;
    static std::mutex mu;
    MapKey k;
    memset(&k, 0, sizeof(k));
    k.dtype = static_cast<int>(dtype);
    k.rank = static_cast<int>(rank);
    k.swizzle = static_cast<int>(swz);
    k.promo = static_cast<int>(promo);
    k.base = base;
    for (cuuint32_t i = 0; i < rank && i < 5; ++i) {
        k.dims[i] = dims[i];
        k.box[i] = box[i];
        if (i + 1 < rank) k.strides[i] = strides[i];
    }
    bool unit_estr = true;
    for (cuuint32_t i = 0; i < rank; ++i) unit_estr = unit_estr && estr[i] == 1;
    std::lock_guard<std::mutex> lk(mu);
    if (unit_estr)
        for (int i = 0; i < kSlots; ++i)
            if (used[i] && keys[i] == k) {
                *map = maps[i];
                return CUDA_SUCCESS;
            }
    CUresult r = enc(map, dtype, rank, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, promo,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r == CUDA_SUCCESS && unit_estr) {
        keys[next] = k;
        maps[next] = *map;
        used[next] = true;
        next = (next + 1) % kSlots;
    }
    return r;
}

// 2-D 16-bit tensor [rows][cols] (cols contiguous; bf16, or f16 when f16), box
// box_cols x box_rows, 128B swizzle.
bool encode_2d_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                    uint32_t box_rows, bool f16 = false)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = encode_cached(enc, map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                     const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
    return r == CUDA_SUCCESS;
}

// 4-D 16-bit NHWC tensor (C innermost; bf16, or f16 when f16), box[4] inner
// first, no swizzle, zero fill.
bool encode_nhwc_h16(CUtensorMap* map, const void* base, uint64_t N, uint64_t H, uint64_t W, uint64_t C,
                     const unsigned box[4], bool f16)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {C, W, H, N};
    const cuuint64_t strides[3] = {C * 2, W * C * 2, H * W * C * 2};
    const cuuint32_t b[4] = {box[0], box[1], box[2], box[3]};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = encode_cached(enc, map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                     const_cast<void*>(base), dims, strides, b, estr, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B);
    return r == CUDA_SUCCESS;
}

// 4-D bf16 planar tensor [C][Y][N][Xs] seen as dims (X, N, Y, C) inner first,
// box (64, 8, nr, 1), 128-byte swizzle, zero fill outside the tensor.
bool encode_planar_bf16(CUtensorMap* map, const void* base, uint64_t X, uint64_t N, uint64_t Y, uint64_t C,
                        uint64_t Xs, unsigned nr)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {X, N, Y, C};
    const cuuint64_t strides[3] = {Xs * 2, N * Xs * 2, Y * N * Xs * 2};
    const cuuint32_t b[4] = {64, 8, nr, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = encode_cached(enc, map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, b, estr, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B);
    return r == CUDA_SUCCESS;
}

// Maps of the depthwise transposes (128-byte swizzle, box rows of 64 elements):
// NHWC (dims C, W, H, N) with a box of 64 channels by 64 positions along W
// (orientation 0) or H (orientation 1), and planar [C][Y][N][Xs] (dims X, N, Y, C)
// with a box of 64 x by 64 c.
bool encode_nhwc_tr(CUtensorMap* map, const void* base, uint64_t N, uint64_t H, uint64_t W, uint64_t C, int orient)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {C, W, H, N};
    const cuuint64_t strides[3] = {C * 2, W * C * 2, H * W * C * 2};
    const cuuint32_t b[4] = {64, orient ? 1u : 64u, orient ? 64u : 1u, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return encode_cached(enc, map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, b, estr, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) == CUDA_SUCCESS;
}

bool encode_planar_tr(CUtensorMap* map, const void* base, uint64_t X, uint64_t N, uint64_t Y, uint64_t C, uint64_t Xs)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {X, N, Y, C};
    const cuuint64_t strides[3] = {Xs * 2, N * Xs * 2, Y * N * Xs * 2};
    const cuuint32_t b[4] = {64, 1, 1, 64};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return encode_cached(enc, map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, b, estr, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) == CUDA_SUCCESS;
}

// The planar dX of the tensor-core depthwise path as the MMA epilogue stores it:
// dims (X, N, Y, C) of [C][Y][N][Xs], box (64, 8, 8, 1), no swizzle.
bool encode_planar_store(CUtensorMap* map, const void* base, uint64_t X, uint64_t N, uint64_t Y, uint64_t C, uint64_t Xs)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {X, N, Y, C};
    const cuuint64_t strides[3] = {Xs * 2, N * Xs * 2, Y * N * Xs * 2};
    const cuuint32_t b[4] = {64, 8, 8, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return encode_cached(enc, map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, b, estr, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int env_int(const char* name, int dflt)
{
    const char* v = dgrad::tuning_env(name);
    return v && *v ? atoi(v) : dflt;
}

// Checks shared by both entry points.  Fills the output extents.
dgrad_status_t validate_common(const dgrad_problem_t* p, dgrad_dtype_t dtype, int64_t* Ho, int64_t* Wo,
                               int* pad_w)
{
    if (!p) return DGRAD_ERR_INVALID;
    if (dtype != DGRAD_F32 && dtype != DGRAD_BF16 && dtype != DGRAD_F16) return DGRAD_ERR_INVALID;
    if (p->N < 0 || p->H < 1 || p->W < 1 || p->C < 1 || p->K < 1) return DGRAD_ERR_INVALID;
    if (p->KH < 1 || p->KW < 1 || p->stride < 1) return DGRAD_ERR_INVALID;
    if (p->pad_h < 0 || p->pad_w < -1) return DGRAD_ERR_INVALID;
    const int pw = p->pad_w == -1 ? p->pad_h : p->pad_w;
    const int64_t nh = p->H + 2 * static_cast<int64_t>(p->pad_h) - p->KH;
    const int64_t nw = p->W + 2 * static_cast<int64_t>(pw) - p->KW;
    if (nh < 0 || nw < 0) return DGRAD_ERR_INVALID;
    *Ho = nh / p->stride + 1;
    *Wo = nw / p->stride + 1;
    *pad_w = pw;
    return DGRAD_OK;
}

}  // namespace

namespace dgrad {
int device_sm_count()
{
    DeviceState* st = nullptr;
    return device_state(&st) == DGRAD_OK ? st->sms : 148;
}
}  // namespace dgrad

extern "C" {

dgrad_status_t dgrad_out_dims(const dgrad_problem_t* prob, int64_t* Ho, int64_t* Wo)
{
    if (!Ho || !Wo) return DGRAD_ERR_INVALID;
    int pw = 0;
    return validate_common(prob, DGRAD_F32, Ho, Wo, &pw);
}

dgrad_status_t dgrad_pointwise(const dgrad_problem_t* prob, dgrad_dtype_t dtype, const void* dY, const void* W,
                               void* dX, void* stream)
{
    int64_t Ho = 0, Wo = 0;
    int pw = 0;
    dgrad_status_t s = validate_common(prob, dtype, &Ho, &Wo, &pw);
    if (s != DGRAD_OK) return s;
    if (prob->KH != 1 || prob->KW != 1 || prob->stride != 1 || prob->pad_h != 0 || pw != 0)
        return DGRAD_ERR_UNSUPPORTED;
    if (dtype == DGRAD_F16) return dgrad_grouped(prob, 1, dtype, dY, W, dX, stream);   // 1x1 through the tap kernel
    const int64_t M = prob->N * prob->H * prob->W;
    if (M == 0) return DGRAD_OK;
    if (!dY || !W || !dX) return DGRAD_ERR_INVALID;
    const int64_t esz = dtype == DGRAD_BF16 ? 2 : 4;
    if (!aligned16(dY) || !aligned16(W) || !aligned16(dX) || (prob->K * esz) % 16 || (prob->C * esz) % 16)
        return DGRAD_ERR_ALIGNMENT;
    if (M > 0x7FFFFFFFLL || prob->K > 65536 || prob->C > 65536) return DGRAD_ERR_UNSUPPORTED;

    DeviceState* st = nullptr;
    s = device_state(&st);
    if (s != DGRAD_OK) return s;
    dgrad::PwArgs a{M, prob->K, prob->C, dY, W, dX, st->status};
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dtype == DGRAD_F32) {
        e = dgrad::launch_pointwise_f32(a, cs);
    } else {
        CUtensorMap map_a, map_b;
        if (!encode_2d_bf16(&map_a, dY, static_cast<uint64_t>(M), static_cast<uint64_t>(prob->K), 64, 128) ||
            !encode_2d_bf16(&map_b, W, static_cast<uint64_t>(prob->K), static_cast<uint64_t>(prob->C), 64, 64))
            return cuda_fail(cudaErrorInvalidValue);
        // Kernel choice: the SM-pair kernel by default (256-column pair tiles when C > 128);
        // DGRAD_PW_MODE = resident | stream selects the one-SM kernels.
        const char* mode = dgrad::tuning_env("DGRAD_PW_MODE");
        const bool want_stream = mode && strcmp(mode, "stream") == 0;
        const bool want_resident = mode && strcmp(mode, "resident") == 0;
        if (!want_stream && !want_resident) {
            CUtensorMap map_d;
            if (!encode_2d_bf16(&map_d, dX, static_cast<uint64_t>(M), static_cast<uint64_t>(prob->C), 64, 128))
                return cuda_fail(cudaErrorInvalidValue);
            const int bn = env_int("DGRAD_PW_BN", prob->C > 128 ? 256 : 128);
            e = dgrad::launch_pointwise_tc_pair(a, map_a, map_b, map_d, bn, st->sms, cs);
        } else if (want_resident && dgrad::pointwise_tc_resident_ok(a, st->sms)) {
            CUtensorMap map_d;
            if (!encode_2d_bf16(&map_d, dX, static_cast<uint64_t>(M), static_cast<uint64_t>(prob->C), 64, 128))
                return cuda_fail(cudaErrorInvalidValue);
            e = dgrad::launch_pointwise_tc_resident(a, map_a, map_b, map_d, st->sms, cs);
        } else {
            const int bn = env_int("DGRAD_PW_BN", prob->C <= 64 ? 64 : 128);
            e = dgrad::launch_pointwise_tc(a, map_a, map_b, bn, st->sms, cs);
        }
    }
    return e == cudaSuccess ? DGRAD_OK : cuda_fail(e);
}

// Shared checks for the split-K entry points: pointwise shape class, bf16 or f16,
// the problem extents the kernels index with 32-bit integers.
static dgrad_status_t splitk_prepare(const dgrad_problem_t* prob, dgrad_dtype_t dtype, int splits,
                                     dgrad::PwArgs* a, int* sms)
{
    int64_t Ho = 0, Wo = 0;
    int pw = 0;
    dgrad_status_t s = validate_common(prob, dtype, &Ho, &Wo, &pw);
    if (s != DGRAD_OK) return s;
    if (prob->KH != 1 || prob->KW != 1 || prob->stride != 1 || prob->pad_h != 0 || pw != 0)
        return DGRAD_ERR_UNSUPPORTED;
    if (dtype != DGRAD_BF16 && dtype != DGRAD_F16) return DGRAD_ERR_UNSUPPORTED;
    if (splits < 0 || splits > 64) return DGRAD_ERR_INVALID;
    const int64_t M = prob->N * prob->H * prob->W;
    if (M > 0x7FFFFFFFLL || prob->K > 65536 || prob->C > 65536) return DGRAD_ERR_UNSUPPORTED;
    if ((prob->K * 2) % 16 || (prob->C * 2) % 16) return DGRAD_ERR_ALIGNMENT;
    *a = dgrad::PwArgs{M, prob->K, prob->C, nullptr, nullptr, nullptr, nullptr, dtype == DGRAD_F16};
    *sms = 0;
    return DGRAD_OK;
}

dgrad_status_t dgrad_pointwise_splitk_workspace(const dgrad_problem_t* prob, int splits, size_t* bytes,
                                                int* splits_used)
{
    if (!bytes) return DGRAD_ERR_INVALID;
    dgrad::PwArgs a{};
    int sms = 0;
    dgrad_status_t s = splitk_prepare(prob, DGRAD_BF16, splits, &a, &sms);
    if (s != DGRAD_OK) return s;
    if (splits == 0) {
        DeviceState* st = nullptr;
        s = device_state(&st);
        if (s != DGRAD_OK) return s;
        splits = dgrad::pointwise_splitk_auto(a, st->sms);
    }
    *bytes = dgrad::pointwise_splitk_workspace_bytes(a, splits);
    if (splits_used) *splits_used = splits;
    return DGRAD_OK;
}

dgrad_status_t dgrad_pointwise_splitk(const dgrad_problem_t* prob, dgrad_dtype_t dtype, int splits, const void* dY,
                                      const void* W, void* dX, void* workspace, size_t workspace_bytes,
                                      void* stream)
{
    dgrad::PwArgs a{};
    int sms = 0;
    dgrad_status_t s = splitk_prepare(prob, dtype, splits, &a, &sms);
    if (s != DGRAD_OK) return s;
    if (a.M == 0) return DGRAD_OK;
    if (!dY || !W || !dX || !workspace) return DGRAD_ERR_INVALID;
    if (!aligned16(dY) || !aligned16(W) || !aligned16(dX) || !aligned16(workspace)) return DGRAD_ERR_ALIGNMENT;
    if (splits > 0 && workspace_bytes < dgrad::pointwise_splitk_workspace_bytes(a, splits)) return DGRAD_ERR_INVALID;
    DeviceState* st = nullptr;
    s = device_state(&st);
    if (s != DGRAD_OK) return s;
    if (splits == 0) splits = dgrad::pointwise_splitk_auto(a, st->sms);
    if (workspace_bytes < dgrad::pointwise_splitk_workspace_bytes(a, splits)) return DGRAD_ERR_INVALID;
    a.dY = dY;
    a.W = W;
    a.dX = dX;
    a.status = st->status;
    CUtensorMap map_a, map_b;
    if (!encode_2d_bf16(&map_a, dY, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.K), 64, 128, a.f16) ||
        !encode_2d_bf16(&map_b, W, static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.C), 64, 64, a.f16))
        return cuda_fail(cudaErrorInvalidValue);
    cudaError_t e = dgrad::launch_pointwise_tc_splitk(a, map_a, map_b, splits, static_cast<float*>(workspace),
                                                       st->sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DGRAD_OK : cuda_fail(e);
}

dgrad_status_t dgrad_grouped(const dgrad_problem_t* prob, int64_t groups, dgrad_dtype_t dtype, const void* dY,
                             const void* W, void* dX, void* stream)
{
    int64_t Ho = 0, Wo = 0;
    int pw = 0;
    dgrad_status_t s = validate_common(prob, dtype, &Ho, &Wo, &pw);
    if (s != DGRAD_OK) return s;
    if (groups < 1 || prob->K % groups || prob->C % groups) return DGRAD_ERR_INVALID;
    if (dtype == DGRAD_F32) return DGRAD_ERR_UNSUPPORTED;
    if (prob->KH > 64 || prob->KW > 64 || prob->stride > 64) return DGRAD_ERR_UNSUPPORTED;
    if (prob->K > 65536 || prob->C > 65536 || prob->H > (1 << 24) || prob->W > (1 << 24) || prob->N > (1 << 24))
        return DGRAD_ERR_UNSUPPORTED;
    const int64_t Kg = prob->K / groups;
    const int64_t Cg = prob->C / groups;
    if (prob->N == 0) return DGRAD_OK;
    if (!dY || !W || !dX) return DGRAD_ERR_INVALID;
    if (!aligned16(dY) || !aligned16(W) || !aligned16(dX) || (Kg * 2) % 16 || (Cg * 2) % 16)
        return DGRAD_ERR_ALIGNMENT;
    DeviceState* st = nullptr;
    s = device_state(&st);
    if (s != DGRAD_OK) return s;
    dgrad::DenseArgs d{};
    d.dX = dX;
    d.status = st->status;
    d.N = static_cast<int>(prob->N);
    d.H = static_cast<int>(prob->H);
    d.W = static_cast<int>(prob->W);
    d.C = static_cast<int>(prob->C);
    d.K = static_cast<int>(prob->K);
    d.Ho = static_cast<int>(Ho);
    d.Wo = static_cast<int>(Wo);
    d.KH = prob->KH;
    d.KW = prob->KW;
    d.S = prob->stride;
    d.ph = prob->pad_h;
    d.pw = pw;
    d.G = static_cast<int>(groups);
    d.Kg = static_cast<int>(Kg);
    d.Cg = static_cast<int>(Cg);
    d.f16 = dtype == DGRAD_F16;
    dgrad::plan_dense(&d);
    auto enc = tensor_map_encoder();
    if (!enc) return cuda_fail(cudaErrorInvalidValue);
    const CUtensorMapDataType ty = d.f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUtensorMap map_a, map_b;
    {
        // dY as (Kg, G, Wo, Ho, N)
        const cuuint64_t dims[5] = {static_cast<cuuint64_t>(Kg), static_cast<cuuint64_t>(groups),
                                    static_cast<cuuint64_t>(Wo), static_cast<cuuint64_t>(Ho),
                                    static_cast<cuuint64_t>(prob->N)};
        const cuuint64_t kb = static_cast<cuuint64_t>(prob->K) * 2;
        const cuuint64_t strides[4] = {static_cast<cuuint64_t>(Kg) * 2, kb, kb * dims[2], kb * dims[2] * dims[3]};
        const cuuint32_t box[5] = {64, 1, 16, 8, 1};
        const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
        if (encode_cached(enc, &map_a, ty, 5, const_cast<void*>(dY), dims, strides, box, estr, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) != CUDA_SUCCESS)
            return cuda_fail(cudaErrorInvalidValue);
    }
    {
        // W [KH][KW][K][Cg] as (Cg, Kg, G, KH*KW)
        const cuuint64_t dims[4] = {static_cast<cuuint64_t>(Cg), static_cast<cuuint64_t>(Kg),
                                    static_cast<cuuint64_t>(groups),
                                    static_cast<cuuint64_t>(prob->KH) * static_cast<cuuint64_t>(prob->KW)};
        const cuuint64_t strides[3] = {dims[0] * 2, dims[0] * dims[1] * 2, dims[0] * dims[1] * dims[2] * 2};
        const cuuint32_t box[4] = {64, 64, 1, 1};
        const cuuint32_t estr[4] = {1, 1, 1, 1};
        if (encode_cached(enc, &map_b, ty, 4, const_cast<void*>(W), dims, strides, box, estr, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) != CUDA_SUCCESS)
            return cuda_fail(cudaErrorInvalidValue);
    }
    const int bn = env_int("DGRAD_DENSE_BN", Cg <= 64 ? 64 : 128);
    cudaError_t e = dgrad::launch_dense_tc(d, map_a, map_b, bn, st->sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DGRAD_OK : cuda_fail(e);
}

dgrad_status_t dgrad_dense(const dgrad_problem_t* prob, dgrad_dtype_t dtype, const void* dY, const void* W, void* dX,
                           void* stream)
{
    return dgrad_grouped(prob, 1, dtype, dY, W, dX, stream);
}

// Shared checks for the tensor-core depthwise entry points: stride-1 depthwise,
// bf16, extents within the kernels' 32-bit indexing and grid limits, and a tile
// plan that fits one SM.
static dgrad_status_t toeplitz_prepare(const dgrad_problem_t* prob, dgrad_dtype_t dtype, dgrad::DwArgs* a,
                                       dgrad::ToepPlan* plan, bool nhwc)
{
    int64_t Ho = 0, Wo = 0;
    int pw = 0;
    dgrad_status_t s = validate_common(prob, dtype, &Ho, &Wo, &pw);
    if (s != DGRAD_OK) return s;
    if ((dtype != DGRAD_BF16 && dtype != DGRAD_F16) || prob->stride != 1 || prob->K != prob->C)
        return DGRAD_ERR_UNSUPPORTED;
    if (prob->KH > 64 || prob->KW > 64) return DGRAD_ERR_UNSUPPORTED;
    if (prob->pad_h > prob->KH - 1 || pw > prob->KW - 1) return DGRAD_ERR_UNSUPPORTED;
    if ((prob->C * 2) % 16) return DGRAD_ERR_ALIGNMENT;
    if (prob->N > 65535 || prob->H > 65535 || prob->W > 65535 || prob->C > (1 << 24)) return DGRAD_ERR_UNSUPPORTED;
    *a = dgrad::DwArgs{};
    a->N = static_cast<int>(prob->N);
    a->H = static_cast<int>(prob->H);
    a->W = static_cast<int>(prob->W);
    a->C = static_cast<int>(prob->C);
    a->Ho = static_cast<int>(Ho);
    a->Wo = static_cast<int>(Wo);
    a->KH = prob->KH;
    a->KW = prob->KW;
    a->S = 1;
    a->ph = prob->pad_h;
    a->pw = pw;
    a->bf16 = dtype == DGRAD_BF16;
    a->f16 = dtype == DGRAD_F16;
    if (!dgrad::plan_dw_toeplitz(*a, plan, nhwc)) return DGRAD_ERR_UNSUPPORTED;
    return DGRAD_OK;
}



dgrad_status_t dgrad_depthwise_tc_workspace(const dgrad_problem_t* prob, size_t* bytes)
{
    if (!bytes) return DGRAD_ERR_INVALID;
    dgrad::DwArgs a{};
    dgrad::ToepPlan plan{};
    dgrad_status_t s = toeplitz_prepare(prob, DGRAD_BF16, &a, &plan, false);
    if (s != DGRAD_OK) return s;
    *bytes = prob->N == 0 ? 0 : plan.ws_in + plan.ws_out + plan.ws_f;
    return DGRAD_OK;
}

dgrad_status_t dgrad_depthwise_tc(const dgrad_problem_t* prob, dgrad_dtype_t dtype, const void* dY, const void* W,
                                  void* dX, void* workspace, size_t workspace_bytes, void* stream)
{
    dgrad::DwArgs a{};
    dgrad::ToepPlan plan{};
    dgrad_status_t s = toeplitz_prepare(prob, dtype, &a, &plan, false);
    if (s != DGRAD_OK) return s;
    if (prob->N == 0) return DGRAD_OK;
    if (!dY || !W || !dX || !workspace) return DGRAD_ERR_INVALID;
    if (!aligned16(dY) || !aligned16(W) || !aligned16(dX) || !aligned16(workspace)) return DGRAD_ERR_ALIGNMENT;
    if (workspace_bytes < plan.ws_in + plan.ws_out + plan.ws_f) return DGRAD_ERR_INVALID;
    DeviceState* st = nullptr;
    s = device_state(&st);
    if (s != DGRAD_OK) return s;
    a.dY = dY;
    a.filt = W;
    a.dX = dX;
    a.status = st->status;
    dgrad::ToepMaps maps{};
    if (!encode_planar_bf16(&maps.b, workspace, static_cast<uint64_t>(plan.Xi), static_cast<uint64_t>(a.N),
                            static_cast<uint64_t>(plan.Yi), static_cast<uint64_t>(a.C),
                            static_cast<uint64_t>(plan.Xsi), static_cast<unsigned>(plan.b_rows)))
        return cuda_fail(cudaErrorInvalidValue);
    // TMA transposes when every map encodes (DGRAD_TC_TRANSPOSE=cuda selects the CUDA-core ones)
    const void* dXp = static_cast<const uint8_t*>(workspace) + plan.ws_in;
    const char* trm = dgrad::tuning_env("DGRAD_TC_TRANSPOSE");
    maps.tma_transpose =
        !(trm && strcmp(trm, "cuda") == 0) &&
        encode_nhwc_tr(&maps.pack_src, dY, static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.Ho),
                       static_cast<uint64_t>(a.Wo), static_cast<uint64_t>(a.C), plan.orient) &&
        encode_planar_tr(&maps.pack_dst, workspace, static_cast<uint64_t>(plan.Xi), static_cast<uint64_t>(a.N),
                         static_cast<uint64_t>(plan.Yi), static_cast<uint64_t>(a.C), static_cast<uint64_t>(plan.Xsi)) &&
        encode_planar_tr(&maps.unpack_src, dXp, static_cast<uint64_t>(plan.Xo), static_cast<uint64_t>(a.N),
                         static_cast<uint64_t>(plan.Yo), static_cast<uint64_t>(a.C), static_cast<uint64_t>(plan.Xso)) &&
        encode_nhwc_tr(&maps.unpack_dst, dX, static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.H),
                       static_cast<uint64_t>(a.W), static_cast<uint64_t>(a.C), plan.orient);
    maps.tma_epi = plan.tma_epi &&
                   encode_planar_store(&maps.d_store, dXp, static_cast<uint64_t>(plan.Xo), static_cast<uint64_t>(a.N),
                                       static_cast<uint64_t>(plan.Yo), static_cast<uint64_t>(a.C),
                                       static_cast<uint64_t>(plan.Xso));
    cudaError_t e = dgrad::launch_dw_toeplitz(a, plan, maps, workspace, st->sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DGRAD_OK : cuda_fail(e);
}

dgrad_status_t dgrad_depthwise(const dgrad_problem_t* prob, dgrad_dtype_t dtype, dgrad_dw_mode_t mode,
                               const void* dY, const void* W, void* dX, void* stream)
{
    int64_t Ho = 0, Wo = 0;
    int pw = 0;
    dgrad_status_t s = validate_common(prob, dtype, &Ho, &Wo, &pw);
    if (s != DGRAD_OK) return s;
    if (mode != DGRAD_DW_AUTO && mode != DGRAD_DW_ROTATED && mode != DGRAD_DW_ROWSTREAM) return DGRAD_ERR_INVALID;
    if (prob->K != prob->C) return DGRAD_ERR_UNSUPPORTED;
    if (prob->KH > 64 || prob->KW > 64) return DGRAD_ERR_UNSUPPORTED;
    if (prob->pad_h > prob->KH - 1 || pw > prob->KW - 1) return DGRAD_ERR_UNSUPPORTED;
    const bool auto_mode = mode == DGRAD_DW_AUTO;
    if (mode == DGRAD_DW_AUTO) mode = prob->stride == 1 ? DGRAD_DW_ROTATED : DGRAD_DW_ROWSTREAM;
    if (mode == DGRAD_DW_ROTATED && prob->stride != 1) return DGRAD_ERR_UNSUPPORTED;
    if (prob->stride > 8) return DGRAD_ERR_UNSUPPORTED;
    if (prob->H > (1 << 24) || prob->W > (1 << 24) || prob->C > (1 << 24)) return DGRAD_ERR_UNSUPPORTED;
    if (prob->N == 0) return DGRAD_OK;
    if (!dY || !W || !dX) return DGRAD_ERR_INVALID;
    const int64_t esz = dtype == DGRAD_F32 ? 4 : 2;
    if (!aligned16(dY) || !aligned16(W) || !aligned16(dX) || (prob->C * esz) % 16) return DGRAD_ERR_ALIGNMENT;

    DeviceState* st = nullptr;
    s = device_state(&st);
    if (s != DGRAD_OK) return s;
    dgrad::DwArgs a{};
    a.N = static_cast<int>(prob->N);
    a.H = static_cast<int>(prob->H);
    a.W = static_cast<int>(prob->W);
    a.C = static_cast<int>(prob->C);
    a.Ho = static_cast<int>(Ho);
    a.Wo = static_cast<int>(Wo);
    a.KH = prob->KH;
    a.KW = prob->KW;
    a.S = prob->stride;
    a.ph = prob->pad_h;
    a.pw = pw;
    a.bf16 = dtype == DGRAD_BF16;
    a.f16 = dtype == DGRAD_F16;
    a.dY = dY;
    a.filt = W;
    a.dX = dX;
    a.status = st->status;
    if (prob->N > 0x7FFFFFFFLL) return DGRAD_ERR_UNSUPPORTED;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    unsigned box[4];
    const char* rk = dgrad::tuning_env("DGRAD_ROT_KERNEL");
    const bool force_line = rk && strcmp(rk, "line") == 0;
    if (auto_mode && prob->stride == 1 && dtype != DGRAD_F32 && prob->KH * prob->KW > 49) {
        // Large stride-1 filters in 16-bit: the tensor-core banded-Toeplitz kernel, when
        // its tile plan fits (else the FP32 kernels below).
        dgrad::ToepPlan plan{};
        if (dgrad::plan_dw_toeplitz(a, &plan, true) && (prob->C % 8) == 0) {
            e = dgrad::launch_dw_toeplitz_nhwc(a, plan, cs);
            if (e != cudaErrorNotSupported) return e == cudaSuccess ? DGRAD_OK : cuda_fail(e);
        }
    }
    if (unsigned tbox_dx[4]; mode == DGRAD_DW_ROTATED && !force_line && dgrad::dw_tile_box(a, box, tbox_dx)) {
        // small filters: one halo tile per CTA
        CUtensorMap map, dx_map;
        if (!encode_nhwc_h16(&map, dY, static_cast<uint64_t>(prob->N), static_cast<uint64_t>(Ho),
                             static_cast<uint64_t>(Wo), static_cast<uint64_t>(prob->C), box, a.f16))
            return cuda_fail(cudaErrorInvalidValue);
        // the output map is optional: without it the kernel stores dX directly
        const bool dx_ok = aligned16(dX) && encode_nhwc_h16(&dx_map, dX, static_cast<uint64_t>(prob->N),
                                                            static_cast<uint64_t>(prob->H), static_cast<uint64_t>(prob->W),
                                                            static_cast<uint64_t>(prob->C), tbox_dx, a.f16);
        e = dgrad::launch_dw_tile(a, map, dx_ok ? &dx_map : nullptr, cs);
    } else if (mode == DGRAD_DW_ROTATED) {
        e = dgrad::launch_dw_rotated(a, cs);
    } else if (unsigned box_dx[4], rows8 = 1;
               env_int("DGRAD_RS_GENERIC", 0) == 0 && dgrad::dw_rowstream_fast_box(a, box, box_dx, &rows8)) {
        CUtensorMap map, dx_map, dx_map8;
        if (!encode_nhwc_h16(&map, dY, static_cast<uint64_t>(prob->N), static_cast<uint64_t>(Ho),
                             static_cast<uint64_t>(Wo), static_cast<uint64_t>(prob->C), box, a.f16))
            return cuda_fail(cudaErrorInvalidValue);
        // the output map is optional: without it the kernel stores dX directly
        const bool dx_ok = aligned16(dX) && encode_nhwc_h16(&dx_map, dX, static_cast<uint64_t>(prob->N),
                                                            static_cast<uint64_t>(prob->H), static_cast<uint64_t>(prob->W),
                                                            static_cast<uint64_t>(prob->C), box_dx, a.f16);
        const unsigned box_dx8[4] = {box_dx[0], box_dx[1], rows8, 1};
        const bool dx8_ok = dx_ok && encode_nhwc_h16(&dx_map8, dX, static_cast<uint64_t>(prob->N),
                                                     static_cast<uint64_t>(prob->H), static_cast<uint64_t>(prob->W),
                                                     static_cast<uint64_t>(prob->C), box_dx8, a.f16);
        e = dgrad::launch_dw_rowstream_fast(a, map, dx8_ok ? &dx_map : nullptr, dx8_ok ? &dx_map8 : nullptr, 0, cs);
    } else {
        e = dgrad::launch_dw_rowstream(a, cs);
    }
    if (e == cudaErrorInvalidConfiguration) return DGRAD_ERR_UNSUPPORTED;
    return e == cudaSuccess ? DGRAD_OK : cuda_fail(e);
}

dgrad_status_t dgrad_check_status(void* stream)
{
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    DeviceState* st = nullptr;
    dgrad_status_t s = device_state(&st);
    if (s != DGRAD_OK) return s;
    int v = 0;
    e = cudaMemcpy(&v, st->status, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e);
    if (v != 0) {
        const int zero = 0;
        e = cudaMemcpy(st->status, &zero, sizeof(int), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return v == dgrad::DEV_TIMEOUT ? DGRAD_ERR_TIMEOUT : v == dgrad::DEV_BOUNDS ? DGRAD_ERR_BOUNDS : DGRAD_OK;
}

const char* dgrad_status_string(dgrad_status_t s)
{
    switch (s) {
    case DGRAD_OK: return "ok";
    case DGRAD_ERR_INVALID: return "invalid argument";
    case DGRAD_ERR_UNSUPPORTED: return "unsupported problem for this entry point";
    case DGRAD_ERR_ALIGNMENT: return "pointer or channel row not 16-byte aligned";
    case DGRAD_ERR_CUDA: return "CUDA error";
    case DGRAD_ERR_TIMEOUT: return "a kernel gave up waiting (timeout)";
    case DGRAD_ERR_BOUNDS: return "a debug-build index check failed (a store was skipped)";
    }
    return "unknown status";
}

int dgrad_last_cuda_error(void) { return t_last_cuda; }

}  // extern "C"

void dgrad::record_cuda_error(cudaError_t e) { t_last_cuda = static_cast<int>(e); }

// ------------------------------------------------------------------ diagnostics

namespace {

// One CTA waits on an mbarrier that nothing will ever complete, with a cycle
// budget; when the budget runs out it records the timeout exactly as the real
// kernels do and returns.
__global__ void selftest_timeout_kernel(long long limit_cycles, int* status)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        dgrad::mbar_init(&bar, 1);
        dgrad::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        bool ok = dgrad::mbar_try_wait(&bar, 0);
        const long long t0 = clock64();
        while (!ok && clock64() - t0 <= limit_cycles) ok = dgrad::mbar_try_wait(&bar, 0);
        if (!ok) dgrad::report_timeout(status);
    }
}

// FMA-rate probe: 8 independent accumulator chains per thread, `iters` rounds.
// packed = 1 uses fma.rn.f32x2 (two FMAs per instruction).  The result is
// written so the work cannot be discarded.
__global__ void __launch_bounds__(256) fma_probe_kernel(int iters, int packed, float* sink)
{
    float a = 1.0f + threadIdx.x * 1e-7f, b = 0.999999f;
    if (packed) {
        float2 acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = make_float2(a + i, a - i);
        const float2 m = make_float2(b, b), c = make_float2(1e-7f, -1e-7f);
        for (int it = 0; it < iters; ++it)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = __ffma2_rn(acc[i], m, c);
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) s += acc[i].x + acc[i].y;
        if (s == 12345.678f) sink[blockIdx.x] = s;
    } else {
        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = a + i;
        for (int it = 0; it < iters; ++it)
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] = fmaf(acc[i], b, 1e-7f);
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) s += acc[i];
        if (s == 12345.678f) sink[blockIdx.x] = s;
    }
}

}  // namespace

extern "C" {

dgrad_status_t dgrad_selftest_timeout(long long limit_cycles, void* stream)
{
    if (limit_cycles < 0 || limit_cycles > dgrad::kWaitCycles) return DGRAD_ERR_INVALID;
    DeviceState* st = nullptr;
    dgrad_status_t s = device_state(&st);
    if (s != DGRAD_OK) return s;
    selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles, st->status);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DGRAD_OK : cuda_fail(e);
}

dgrad_status_t dgrad_fma_probe(int blocks, int iters, int packed, float* sink, void* stream)
{
    if (blocks < 1 || iters < 1 || !sink) return DGRAD_ERR_INVALID;
    fma_probe_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(iters, packed, sink);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DGRAD_OK : cuda_fail(e);
}

}  // extern "C"
