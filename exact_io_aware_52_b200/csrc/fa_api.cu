// fa_api.cu -- the C ABI declared in include/fa.h: argument validation, the
// per-device property cache, TMA tensor-map encoding and the kernel launch.
// The library allocates nothing: every buffer belongs to the caller.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"
#include "fa_bwd_kernel.cuh"
#include "fa_combine_kernel.cuh"
#include "fa_fwd_d256_kernel.cuh"
#include "fa_fwd_kernel.cuh"

namespace {

constexpr int kVersion = 300;  // 0.3.0
constexpr int kMaxDevices = 64;
constexpr int kMaxSplits = 1024;

// Scheduler slots of the dynamic work distribution (causal forward, backward):
// four words per slot, [0] next unit, [1] CTAs done, [2, 4) the 64-bit owner
// (grid id + 1 of the launch using the slot, 0: free); zero at module load and
// returned to zero by the last CTA of each launch.  A launch takes the next
// slot round-robin; launches that meet on a slot (more than kSchedSlots in
// flight at once, or one CUDA graph replayed on several streams) serialise on
// it in the kernel, and a launch whose wait for its slot outlasts its time
// limit reports FA_ERR_SCHED_BUSY.
constexpr int kSchedSlots = 64;
constexpr int kSchedWords = 4;
static __device__ __align__(16) uint32_t g_sched[kSchedWords * kSchedSlots];
std::atomic<uint32_t> g_sched_next{0};

struct DeviceInfo {
    bool probed = false;
    bool supported = false;
    int num_sms = 0;
    uint32_t *sched = nullptr;  // g_sched on this device
    bool attr_set[4][2] = {};  // [d = 64, 128, 256, 128 with E4M3 inputs][bf16 out]
    bool bwd_attr_set[2] = {};  // backward kernel, [d == 128]
    cudaStream_t copy_in = nullptr, copy_out = nullptr;  // fa_fwd_host's copy streams (created on first use)
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_d(int d) { return d == 64 || d == 128 || d == 256; }

bool e4m3_in(const fa_fwd_params *p) { return p->in_dtype == FA_IN_E4M3; }

bool valid_descale(float x) { return std::isfinite(x) && x >= 0.f; }
float descale(float x) { return x > 0.f ? x : 1.f; }

// Query rows per work unit: two 128-row tiles for d <= 128 (the ping-pong
// kernel), one for d = 256 (the one-tile kernel).
int unit_rows(int d) { return d == 256 ? fa::d256::kUnitRows : fa::kUnitRows; }

fa_status load_encoder() {
    if (g_encode) return FA_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return FA_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return FA_OK;
}

// Device checks are cached per device ordinal.
fa_status probe_device(int *dev_out, DeviceInfo **info_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    DeviceInfo &di = g_dev[dev];
    if (!di.probed) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return FA_ERR_CUDA;
        di.supported = (major == 10 && minor == 0);  // the binary is sm_100a only
        di.num_sms = sms;
        if (di.supported) {
            void *sp = nullptr;
            if (cudaGetSymbolAddress(&sp, g_sched) != cudaSuccess || sp == nullptr) {
                cudaGetLastError();
                return FA_ERR_CUDA;
            }
            di.sched = static_cast<uint32_t *>(sp);
        }
        di.probed = true;
    }
    if (!di.supported) return FA_ERR_UNSUPPORTED;
    *dev_out = dev;
    *info_out = &di;
    return FA_OK;
}

// 3-D map over a contiguous [B*H][N][D] tensor of bf16 (elem_bytes 2) or
// E4M3 (elem_bytes 1, mapped as bytes): dims innermost first {D, N, B*H};
// box {128 / elem_bytes, 128, 1} (one 128-byte column block of a 128-row
// tile); 128-byte swizzle, the layout the tcgen05 descriptors describe.
// Out-of-range rows read as zero.
fa_status encode_map(CUtensorMap *map, const void *base, int BH, int N, int D, int elem_bytes = 2) {
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * elem_bytes, (cuuint64_t)N * D * elem_bytes};
    cuuint32_t box[3] = {(cuuint32_t)(128 / elem_bytes), (cuuint32_t)fa::BM, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = g_encode(map, dt, 3, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// 3-D map over a contiguous [B*H][N][D] fp32 tensor, box {32, 128, 1} (one
// 128-byte column block of a 128-row tile), 128-byte swizzle: the target of
// the backward's dQ reduce-add.
fa_status encode_map_f32(CUtensorMap *map, void *base, int BH, int N, int D) {
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)N * D * 4};
    cuuint32_t box[3] = {32, (cuuint32_t)fa::BM, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// 3-D map over the fp32 output [planes][N][D] (planes = key splits x B x H),
// box {32, 32, 1}, 128-byte swizzle: the d = 64 epilogue's TMA stores of one
// warp's 32 rows, 32 columns per box.  Rows past N are not written.
fa_status encode_map_o32(CUtensorMap *map, void *base, long long planes, int N, int D) {
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)planes};
    cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)N * D * 4};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// Validation that needs no device, except the workspace clause.
fa_status validate_args(const fa_fwd_params *p) {
    if (!p) return FA_ERR_INVALID_ARGUMENT;
    if (p->B < 0 || p->H < 0 || p->N < 0) return FA_ERR_INVALID_ARGUMENT;
    if (!(std::isfinite(p->scale) && p->scale > 0.f)) return FA_ERR_INVALID_ARGUMENT;
    if (p->causal != 0 && p->causal != 1) return FA_ERR_INVALID_ARGUMENT;
    if (p->o_dtype != FA_O_F32 && p->o_dtype != FA_O_BF16) return FA_ERR_INVALID_ARGUMENT;
    if (p->flags & ~FA_FLAG_EAGER_RESCALE) return FA_ERR_INVALID_ARGUMENT;
    if (p->H_kv < 0 || (p->H_kv > 0 && p->H % p->H_kv != 0)) return FA_ERR_INVALID_ARGUMENT;
    if (p->N_k < 0 || p->num_splits < 0 || p->num_splits > kMaxSplits) return FA_ERR_INVALID_ARGUMENT;
    if (p->in_dtype != FA_IN_BF16 && p->in_dtype != FA_IN_E4M3) return FA_ERR_INVALID_ARGUMENT;
    if (!valid_descale(p->descale_q) || !valid_descale(p->descale_k) || !valid_descale(p->descale_v))
        return FA_ERR_INVALID_ARGUMENT;
    if (p->test_drop_load < 0) return FA_ERR_INVALID_ARGUMENT;
    if (!supported_d(p->d)) return FA_ERR_UNSUPPORTED;
    if (e4m3_in(p) && p->d != 128) return FA_ERR_UNSUPPORTED;
    const long long rows = (long long)p->B * p->H * p->N;
    if (rows == 0) return FA_OK;
    if ((long long)p->B * p->H > 0x7fffffffLL || (long long)p->B * p->H * ((p->N + 127) / 128) > 0x7fffffffLL)
        return FA_ERR_INVALID_ARGUMENT;
    if (!p->q || !p->k || !p->v || !p->o || !p->lse) return FA_ERR_INVALID_ARGUMENT;
    if (!aligned16(p->q) || !aligned16(p->k) || !aligned16(p->v) || !aligned16(p->o)) return FA_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(p->lse) & 3u) || (reinterpret_cast<uintptr_t>(p->k_len) & 3u) ||
        (reinterpret_cast<uintptr_t>(p->dev_status) & 3u))
        return FA_ERR_MISALIGNED;
    return FA_OK;
}

// Validation that needs no device: shared by every entry point.
fa_status validate(const fa_fwd_params *p) {
    const fa_status st = validate_args(p);
    if (st != FA_OK || (long long)p->B * p->H * p->N == 0) return st;
    if (p->num_splits > 1) {
        if (!p->workspace || p->workspace_bytes < fa_fwd_workspace_bytes(p)) return FA_ERR_INVALID_ARGUMENT;
        if (!aligned16(p->workspace)) return FA_ERR_MISALIGNED;
    }
    return FA_OK;
}

// Key tiles of 128 keys and the split layout actually used for *p.
struct SplitPlan {
    int n_k;          // keys
    int splits;       // effective split count (no empty trailing splits)
    int split_tiles;  // key tiles per split
};

SplitPlan plan_splits(const fa_fwd_params *p) {
    SplitPlan sp;
    sp.n_k = p->N_k > 0 ? p->N_k : p->N;
    const int tiles = (sp.n_k + fa::BN - 1) / fa::BN;
    int s = p->num_splits > 1 ? p->num_splits : 1;
    if (s > tiles) s = tiles > 0 ? tiles : 1;
    sp.split_tiles = tiles > 0 ? (tiles + s - 1) / s : 1;
    sp.splits = tiles > 0 ? (tiles + sp.split_tiles - 1) / sp.split_tiles : 1;
    return sp;
}

template <int D, bool BF16>
fa_status launch_combine(const float *o_part, const float *lse_part, void *o, float *lse, int splits, long long rows,
                         int num_sms, cudaStream_t stream) {
    const long long warps = rows;
    long long blocks = (warps * 32 + 255) / 256;
    if (blocks > 8LL * num_sms) blocks = 8LL * num_sms;
    fa::fa_combine_kernel<D, BF16><<<(int)blocks, 256, 0, stream>>>(o_part, lse_part, o, lse, splits, rows);
    return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, bool BF16, bool F8 = false>
fa_status launch(const fa::FwdParams &kp, DeviceInfo &di, int grid, cudaStream_t stream) {
    constexpr bool kD256 = D == 256;
    constexpr int kD = kD256 ? 128 : D;
    auto kern = kD256 ? fa::fa_fwd_onetile_kernel<256, BF16> : fa::fa_fwd_sm100_kernel<kD, BF16, F8>;
    const int smem = kD256 ? fa::d256::Cfg1<256>::kSmemBytes : fa::Cfg<kD, F8>::kSmemBytes;
    const int threads = kD256 ? fa::d256::kThreads : fa::kThreads;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        bool &set = di.attr_set[F8 ? 3 : (D == 64 ? 0 : (D == 128 ? 1 : 2))][BF16];
        if (!set) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
                return FA_ERR_CUDA;
            set = true;
        }
    }
    kern<<<grid, threads, smem, stream>>>(kp);
    return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <bool BF16>
fa_status launch_d(int d, bool e4m3, const fa::FwdParams &kp, DeviceInfo &di, int grid, cudaStream_t stream) {
    if (e4m3) return launch<128, BF16, true>(kp, di, grid, stream);
    if (d == 64) return launch<64, BF16>(kp, di, grid, stream);
    if (d == 128) return launch<128, BF16>(kp, di, grid, stream);
    return launch<256, BF16>(kp, di, grid, stream);
}

template <bool BF16>
fa_status launch_combine_d(int d, const float *o_part, const float *lse_part, void *o, float *lse, int splits,
                           long long rows, int num_sms, cudaStream_t stream) {
    if (d == 64) return launch_combine<64, BF16>(o_part, lse_part, o, lse, splits, rows, num_sms, stream);
    if (d == 128) return launch_combine<128, BF16>(o_part, lse_part, o, lse, splits, rows, num_sms, stream);
    return launch_combine<256, BF16>(o_part, lse_part, o, lse, splits, rows, num_sms, stream);
}

fa_status validate_bwd(const fa_bwd_params *p) {
    if (!p) return FA_ERR_INVALID_ARGUMENT;
    if (p->B < 0 || p->H < 0 || p->N < 0 || p->N_k < 0) return FA_ERR_INVALID_ARGUMENT;
    if (!(std::isfinite(p->scale) && p->scale > 0.f)) return FA_ERR_INVALID_ARGUMENT;
    if (p->causal != 0 && p->causal != 1) return FA_ERR_INVALID_ARGUMENT;
    if (p->o_dtype != FA_O_F32 && p->o_dtype != FA_O_BF16) return FA_ERR_INVALID_ARGUMENT;
    if (p->H_kv < 0 || (p->H_kv > 0 && p->H % p->H_kv != 0)) return FA_ERR_INVALID_ARGUMENT;
    if (p->d != 64 && p->d != 128) return FA_ERR_UNSUPPORTED;
    const long long rows = (long long)p->B * p->H * p->N;
    if (rows == 0) return FA_OK;
    const int H_kv = p->H_kv > 0 ? p->H_kv : p->H;
    const int n_k = p->N_k > 0 ? p->N_k : p->N;
    if ((long long)p->B * H_kv * ((n_k + 127) / 128) > 0x7fffffffLL || (long long)p->B * p->H > 0x7fffffffLL)
        return FA_ERR_INVALID_ARGUMENT;
    if (!p->q || !p->k || !p->v || !p->o || !p->dout || !p->lse || !p->dq || !p->dk || !p->dv)
        return FA_ERR_INVALID_ARGUMENT;
    if (!p->workspace || p->workspace_bytes < (size_t)rows * sizeof(float)) return FA_ERR_INVALID_ARGUMENT;
    if (!aligned16(p->q) || !aligned16(p->k) || !aligned16(p->v) || !aligned16(p->o) || !aligned16(p->dout) ||
        !aligned16(p->dq) || !aligned16(p->dk) || !aligned16(p->dv) || !aligned16(p->workspace) ||
        !aligned16(p->lse))
        return FA_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(p->k_len) & 3u) || (reinterpret_cast<uintptr_t>(p->dev_status) & 3u))
        return FA_ERR_MISALIGNED;
    return FA_OK;
}

template <int D>
fa_status launch_bwd(const fa::bwd::BwdParams &kp, const fa_bwd_params *p, DeviceInfo &di, cudaStream_t s) {
    const long long rows = (long long)p->B * p->H * p->N;
    long long blocks = (rows * 32 + 255) / 256;
    if (blocks > 8LL * di.num_sms) blocks = 8LL * di.num_sms;
    if (p->o_dtype == FA_O_BF16)
        fa::fa_bwd_prep_kernel<D, true><<<(int)blocks, 256, 0, s>>>(
            p->o, static_cast<const uint16_t *>(p->dout), static_cast<float *>(p->workspace), p->dq, rows);
    else
        fa::fa_bwd_prep_kernel<D, false><<<(int)blocks, 256, 0, s>>>(
            p->o, static_cast<const uint16_t *>(p->dout), static_cast<float *>(p->workspace), p->dq, rows);
    if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
    auto kern = fa::fa_bwd_sm100_kernel<D>;
    const int smem = fa::bwd::BCfg<D>::kSmemBytes;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        bool &set = di.bwd_attr_set[D == 128];
        if (!set) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
                return FA_ERR_CUDA;
            set = true;
        }
    }
    const int grid = kp.n_units < di.num_sms ? kp.n_units : di.num_sms;
    kern<<<grid, fa::bwd::kThreads, smem, s>>>(kp);
    return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

namespace fa_detail {

fa_status validate_args(const fa_fwd_params *p) { return ::validate_args(p); }

fa_status probe_current_device() {
    int dev = 0;
    DeviceInfo *di = nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    return probe_device(&dev, &di);
}

}  // namespace fa_detail

extern "C" {

size_t fa_bwd_workspace_bytes(const fa_bwd_params *p) {
    if (!p || p->B <= 0 || p->H <= 0 || p->N <= 0) return 0;
    return (size_t)p->B * p->H * p->N * sizeof(float);
}

fa_status fa_bwd(const fa_bwd_params *p, void *stream) {
    fa_status st = validate_bwd(p);
    if (st != FA_OK) return st;
    if ((long long)p->B * p->H * p->N == 0) return FA_OK;
    int dev = 0;
    DeviceInfo *di = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        st = probe_device(&dev, &di);
        if (st == FA_OK) st = load_encoder();
    }
    if (st != FA_OK) return st;
    fa::bwd::BwdParams kp;
    std::memset(&kp, 0, sizeof kp);
    const int BH = p->B * p->H;
    const int H_kv = p->H_kv > 0 ? p->H_kv : p->H;
    const int n_k = p->N_k > 0 ? p->N_k : p->N;
    if ((st = encode_map(&kp.tm_q, p->q, BH, p->N, p->d)) != FA_OK) return st;
    if ((st = encode_map(&kp.tm_do, p->dout, BH, p->N, p->d)) != FA_OK) return st;
    if ((st = encode_map(&kp.tm_k, p->k, p->B * H_kv, n_k, p->d)) != FA_OK) return st;
    if ((st = encode_map(&kp.tm_v, p->v, p->B * H_kv, n_k, p->d)) != FA_OK) return st;
    if ((st = encode_map_f32(&kp.tm_dq, p->dq, BH, p->N, p->d)) != FA_OK) return st;
    kp.lse = p->lse;
    kp.delta = static_cast<const float *>(p->workspace);
    kp.dq = p->dq;
    kp.dk = p->dk;
    kp.dv = p->dv;
    kp.k_len = p->k_len;
    kp.status = p->dev_status;
    kp.B = p->B;
    kp.H = p->H;
    kp.N = p->N;
    kp.Nk = n_k;
    kp.H_kv = H_kv;
    kp.group = p->H / H_kv;
    kp.n_kv_tiles = (n_k + fa::BN - 1) / fa::BN;
    kp.n_units = p->B * H_kv * kp.n_kv_tiles;
    {
        // band of key tiles: the (key/value head, key tile) units in flight
        // (one per SM) should span few enough heads for their Q and dO (~64 MB)
        // to stay in L2
        const double qdo_head = 4.0 * p->N * p->d * (double)(p->H / H_kv);
        int heads_fit = (int)(64.0e6 / (qdo_head > 1.0 ? qdo_head : 1.0));
        if (heads_fit < 1) heads_fit = 1;
        int band = (di->num_sms + heads_fit - 1) / heads_fit;
        kp.band_tiles = band < 1 ? 1 : (band > kp.n_kv_tiles ? kp.n_kv_tiles : band);
    }
    kp.sched = di->sched + kSchedWords * (g_sched_next.fetch_add(1, std::memory_order_relaxed) % kSchedSlots);
    kp.causal = p->causal;
    kp.scale = p->scale;
    kp.scale_log2 = (float)((double)p->scale * 1.4426950408889634074);
    kp.timeout_ns = (uint64_t)(p->timeout_ms ? p->timeout_ms : 2000u) * 1000000ull;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return p->d == 64 ? launch_bwd<64>(kp, p, *di, s) : launch_bwd<128>(kp, p, *di, s);
}


fa_status fa_fwd_ex(const fa_fwd_params *p, void *stream) {
    fa_status st = validate(p);
    if (st != FA_OK) return st;
    if ((long long)p->B * p->H * p->N == 0) return FA_OK;

    int dev = 0;
    DeviceInfo *di = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        st = probe_device(&dev, &di);
        if (st == FA_OK) st = load_encoder();
    }
    if (st != FA_OK) return st;

    fa::FwdParams kp;
    std::memset(&kp, 0, sizeof kp);
    const int BH = p->B * p->H;
    const int H_kv = p->H_kv > 0 ? p->H_kv : p->H;
    const SplitPlan sp = plan_splits(p);
    const int eb = e4m3_in(p) ? 1 : 2;
    if ((st = encode_map(&kp.tm_q, p->q, BH, p->N, p->d, eb)) != FA_OK) return st;
    // a map over zero keys is not encodable; with N_k = 0 no key tile is loaded
    const int n_k_map = sp.n_k > 0 ? sp.n_k : 1;
    if ((st = encode_map(&kp.tm_k, p->k, p->B * H_kv, n_k_map, p->d, eb)) != FA_OK) return st;
    if ((st = encode_map(&kp.tm_v, p->v, p->B * H_kv, n_k_map, p->d, eb)) != FA_OK) return st;
    const long long rows = (long long)BH * p->N;
    float *o_part = nullptr, *lse_part = nullptr;
    if (sp.splits > 1) {  // partials: fp32 [S][rows][d], then fp32 [S][rows]
        o_part = static_cast<float *>(p->workspace);
        lse_part = o_part + (size_t)sp.splits * rows * p->d;
        kp.o = o_part;
        kp.lse = lse_part;
    } else {
        kp.o = p->o;
        kp.lse = p->lse;
    }
    // d = 64 bf16 inputs with fp32 output (or fp32 partials): O leaves through TMA stores
    if (p->d == 64 && !e4m3_in(p) && (sp.splits > 1 || p->o_dtype != FA_O_BF16))
        if ((st = encode_map_o32(&kp.tm_o, kp.o, (long long)sp.splits * BH, p->N, p->d)) != FA_OK) return st;
    kp.k_len = p->k_len;
    kp.status = p->dev_status;
    kp.B = p->B;
    kp.H = p->H;
    kp.N = p->N;
    kp.Nk = sp.n_k;
    kp.group = p->H / H_kv;
    kp.H_kv = H_kv;
    kp.n_blocks = (p->N + unit_rows(p->d) - 1) / unit_rows(p->d);
    kp.n_splits = sp.splits;
    kp.split_tiles = sp.split_tiles;
    kp.n_units = BH * kp.n_blocks * sp.splits;
    {
        // band of query blocks in the unit order: the (query head, block) pairs
        // in flight (about one per SM and split) should span few enough heads
        // for their K and V (~64 MB) to stay in L2
        const double kv_head = 2.0 * sp.n_k * p->d * eb / (double)(p->H / H_kv);
        int heads_fit = (int)(64.0e6 / (kv_head > 1.0 ? kv_head : 1.0));
        if (heads_fit < 1) heads_fit = 1;
        const int in_flight = (di->num_sms + sp.splits - 1) / sp.splits;
        int band = (in_flight + heads_fit - 1) / heads_fit;
        kp.band_blocks = band < 1 ? 1 : (band > kp.n_blocks ? kp.n_blocks : band);
        // causal units differ in cost: hand them out dynamically; key-padded
        // non-causal units differ by batch element: hand them out dynamically,
        // batch elements with the most key tiles first (d <= 128, up to
        // kSortMaxB of them); equal-cost units keep the static snake over
        // head-major order
        kp.sort_b = (!p->causal && p->k_len && p->B <= fa::kSortMaxB && p->d <= 128 && sp.splits == 1) ? 1 : 0;
        kp.dynamic = (p->causal || kp.sort_b) ? 1 : 0;
        if (!p->causal) kp.band_blocks = kp.n_blocks;
    }
    kp.sched = di->sched + kSchedWords * (g_sched_next.fetch_add(1, std::memory_order_relaxed) % kSchedSlots);
    kp.causal = p->causal;
    if (e4m3_in(p)) {
        // value scales: Q K^T by descale_q * descale_k (folded into the softmax
        // scale), O by descale_v.  Weights are 2^(x - m_ref + 7) with x at most
        // tau above m_ref, so they stay at or below 2^(7 + tau) = 430.5 for
        // tau = 1.75, under E4M3's largest finite value 448 (no saturation).
        kp.scale_log2 = (float)((double)p->scale * descale(p->descale_q) * descale(p->descale_k) *
                                1.4426950408889634074);
        kp.tau = (p->flags & FA_FLAG_EAGER_RESCALE) ? 0.f : 1.75f;
        kp.out_scale = descale(p->descale_v);
    } else {
        kp.scale_log2 = (float)((double)p->scale * 1.4426950408889634074);
        kp.tau = (p->flags & FA_FLAG_EAGER_RESCALE) ? 0.f : 8.f;
        kp.out_scale = 1.f;
    }
    kp.timeout_ns = (uint64_t)(p->timeout_ms ? p->timeout_ms : 2000u) * 1000000ull;
    kp.drop_load = p->test_drop_load;

    const int grid = kp.n_units < di->num_sms ? kp.n_units : di->num_sms;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool bf16 = p->o_dtype == FA_O_BF16;
    if (sp.splits > 1) {  // the split pass always writes fp32 partials; the merge writes the output type
        if ((st = launch_d<false>(p->d, e4m3_in(p), kp, *di, grid, s)) != FA_OK) return st;
        return bf16 ? launch_combine_d<true>(p->d, o_part, lse_part, p->o, p->lse, sp.splits, rows, di->num_sms, s)
                    : launch_combine_d<false>(p->d, o_part, lse_part, p->o, p->lse, sp.splits, rows, di->num_sms, s);
    }
    return bf16 ? launch_d<true>(p->d, e4m3_in(p), kp, *di, grid, s)
                : launch_d<false>(p->d, e4m3_in(p), kp, *di, grid, s);
}

size_t fa_fwd_workspace_bytes(const fa_fwd_params *p) {
    if (!p || p->num_splits <= 1 || p->B <= 0 || p->H <= 0 || p->N <= 0 || !supported_d(p->d)) return 0;
    const SplitPlan sp = plan_splits(p);
    if (sp.splits <= 1) return 0;
    const size_t rows = (size_t)p->B * p->H * p->N;
    return (size_t)sp.splits * rows * ((size_t)p->d + 1) * sizeof(float);
}

int fa_fwd_suggest_splits(const fa_fwd_params *p) {
    if (!p || p->B <= 0 || p->H <= 0 || p->N <= 0) return 0;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return 0;
    const int ur = unit_rows(supported_d(p->d) ? p->d : 128);
    const long long units = (long long)p->B * p->H * ((p->N + ur - 1) / ur);
    const long long n_k = p->N_k > 0 ? p->N_k : p->N;
    const long long tiles = (n_k + fa::BN - 1) / fa::BN;
    if (units >= 2LL * sms || tiles <= 1) return 1;
    // Cost model in key-tile steps of one persistent CTA: waves of units times the
    // tiles of the longest split plus a fixed per-unit cost (Q load, drain,
    // epilogue ~ 2 steps), plus the partials' write and re-read (8 (d + 1) bytes
    // per row and split) at ~16 MB of HBM traffic per step across the GPU.
    const double rows = (double)p->B * p->H * p->N;
    const double split_cost = rows * 8.0 * (p->d + 1) / 16.0e6;
    long long best_s = 1;
    double best = 0.0;
    const long long s_max = tiles < kMaxSplits ? tiles : kMaxSplits;
    for (long long s = 1; s <= s_max; ++s) {
        const long long per = (tiles + s - 1) / s;
        const long long eff = (tiles + per - 1) / per;  // splits left after dropping empty ones
        if (eff != s) continue;
        const long long waves = (units * s + sms - 1) / sms;
        const double cost = (double)waves * (double)(per + 2) + (s > 1 ? split_cost * (double)s : 0.0);
        if (s == 1 || cost < best) {
            best = cost;
            best_s = s;
        }
    }
    return (int)best_s;
}

fa_status fa_fwd(const void *q, const void *k, const void *v, float *o, float *lse, int B, int H, int N, int d,
                 int causal, float scale, void *stream) {
    fa_fwd_params p;
    std::memset(&p, 0, sizeof p);
    p.q = q;
    p.k = k;
    p.v = v;
    p.o = o;
    p.lse = lse;
    p.B = B;
    p.H = H;
    p.N = N;
    p.d = d;
    p.causal = causal;
    p.scale = scale;
    p.o_dtype = FA_O_F32;
    return fa_fwd_ex(&p, stream);
}

// fa_fwd_host in one piece: the copies in, the kernel and the copies out,
// one after the other on `stream`.
fa_status host_single(const fa_fwd_host_params *hp, cudaStream_t s) {
    const fa_fwd_params *p = &hp->dev;
    const size_t rows = (size_t)p->B * p->H * p->N;
    const size_t eb = e4m3_in(p) ? 1 : 2;
    const size_t q_bytes = rows * p->d * eb;
    const size_t kv_bytes =
        (size_t)p->B * (p->H_kv > 0 ? p->H_kv : p->H) * (p->N_k > 0 ? p->N_k : p->N) * p->d * eb;
    const size_t o_bytes = rows * p->d * (p->o_dtype == FA_O_BF16 ? 2 : 4);
    if (cudaMemcpyAsync(const_cast<void *>(p->q), hp->q, q_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(const_cast<void *>(p->k), hp->k, kv_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(const_cast<void *>(p->v), hp->v, kv_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return FA_ERR_CUDA;
    if (hp->k_len && cudaMemcpyAsync(const_cast<int32_t *>(p->k_len), hp->k_len, sizeof(int32_t) * p->B,
                                     cudaMemcpyHostToDevice, s) != cudaSuccess)
        return FA_ERR_CUDA;
    fa_status st = fa_fwd_ex(p, s);
    if (st != FA_OK) return st;
    if (cudaMemcpyAsync(hp->o, p->o, o_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemcpyAsync(hp->lse, p->lse, rows * sizeof(float), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return FA_ERR_CUDA;
    return FA_OK;
}

// A piece of a fa_fwd_host call: whole batch elements (B > 1) or, with one
// batch element, whole groups of query heads that share a key/value head.
constexpr int kMaxHostChunks = 8;
struct HostChunk {
    fa_fwd_host_params hp;  // host and device pointers offset to the piece, its shape
    size_t q_bytes, kv_bytes, o_bytes, lse_bytes;
};

// Cuts the call into up to kMaxHostChunks pieces when its copies are large
// (at least 64 MB) and each piece still gives every SM two work units;
// returns the number of pieces (1: keep the call whole).  Such a call is
// bound by the PCIe copies: measured on B200 (B1 H32 N16384 d128 causal),
// 6 pieces 9.67 ms and 13 pieces 9.75 ms against 14.22 ms in one piece.
int host_chunks(const fa_fwd_host_params *hp, int num_sms, HostChunk *out) {
    const fa_fwd_params *p = &hp->dev;
    const int H_kv = p->H_kv > 0 ? p->H_kv : p->H;
    const int group = p->H / H_kv;
    const int n_k = p->N_k > 0 ? p->N_k : p->N;
    const size_t eb = e4m3_in(p) ? 1 : 2, ob = p->o_dtype == FA_O_BF16 ? 2 : 4;
    const size_t rows = (size_t)p->B * p->H * p->N;
    const size_t total = rows * p->d * (eb + ob) + 2 * (size_t)p->B * H_kv * n_k * p->d * eb + rows * 4;
    if (total < ((size_t)64 << 20)) return 1;
    const long long units = (long long)p->B * p->H * ((p->N + unit_rows(p->d) - 1) / unit_rows(p->d)) *
                            (p->num_splits > 1 ? p->num_splits : 1);
    const int dim = p->B > 1 ? p->B : H_kv;  // batch elements, or key/value heads of the one batch element
    int n = dim < kMaxHostChunks ? dim : kMaxHostChunks;
    while (n > 1 && units / n < 2LL * num_sms) --n;
    if (n <= 1) return 1;
    for (int c = 0; c < n; ++c) {
        const int a0 = (int)((long long)dim * c / n), a1 = (int)((long long)dim * (c + 1) / n);
        HostChunk &ch = out[c];
        ch.hp = *hp;
        fa_fwd_params &cp = ch.hp.dev;
        size_t q_off, kv_off, o_off, lse_off;  // elements
        if (p->B > 1) {
            cp.B = a1 - a0;
            q_off = (size_t)a0 * p->H * p->N * p->d;
            kv_off = (size_t)a0 * H_kv * n_k * p->d;
            lse_off = (size_t)a0 * p->H * p->N;
            if (p->k_len) {
                cp.k_len = p->k_len + a0;
                ch.hp.k_len = hp->k_len + a0;
            }
        } else {
            cp.H = (a1 - a0) * group;
            if (p->H_kv > 0) cp.H_kv = a1 - a0;
            q_off = (size_t)a0 * group * p->N * p->d;
            kv_off = (size_t)a0 * n_k * p->d;
            lse_off = (size_t)a0 * group * p->N;
        }
        o_off = q_off;
        cp.q = static_cast<const uint8_t *>(p->q) + q_off * eb;
        cp.k = static_cast<const uint8_t *>(p->k) + kv_off * eb;
        cp.v = static_cast<const uint8_t *>(p->v) + kv_off * eb;
        cp.o = static_cast<uint8_t *>(p->o) + o_off * ob;
        cp.lse = p->lse + lse_off;
        ch.hp.q = static_cast<const uint8_t *>(hp->q) + q_off * eb;
        ch.hp.k = static_cast<const uint8_t *>(hp->k) + kv_off * eb;
        ch.hp.v = static_cast<const uint8_t *>(hp->v) + kv_off * eb;
        ch.hp.o = static_cast<uint8_t *>(hp->o) + o_off * ob;
        ch.hp.lse = hp->lse + lse_off;
        const size_t c_rows = (size_t)cp.B * cp.H * p->N;
        const int c_hkv = cp.H_kv > 0 ? cp.H_kv : cp.H;
        ch.q_bytes = c_rows * p->d * eb;
        ch.kv_bytes = (size_t)cp.B * c_hkv * n_k * p->d * eb;
        ch.o_bytes = c_rows * p->d * ob;
        ch.lse_bytes = c_rows * sizeof(float);
        if (validate(&cp) != FA_OK) return 1;  // a piece the library would refuse: keep the call whole
    }
    return n;
}

// The pieces pipelined over three streams: piece c's copies in on the copy-in
// stream, its kernel on `s` once they have landed, its copies out on the
// copy-out stream once the kernel is done; PCIe carries the two directions at
// once, so the input copies, the kernels and the output copies of different
// pieces overlap.  Returns after `s` has waited for everything.
fa_status host_pipelined(HostChunk *ch, int n, cudaStream_t s, cudaStream_t cin, cudaStream_t cout) {
    cudaEvent_t ev[2 * kMaxHostChunks + 2] = {};
    const int n_ev = 2 * n + 2;
    fa_status st = FA_OK;
    for (int i = 0; i < n_ev && st == FA_OK; ++i)
        if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) st = FA_ERR_CUDA;
    cudaEvent_t start = ev[0], end = ev[1];
    // the caller's earlier work on `s` may still use the device buffers
    if (st == FA_OK && (cudaEventRecord(start, s) != cudaSuccess || cudaStreamWaitEvent(cin, start, 0) != cudaSuccess))
        st = FA_ERR_CUDA;
    for (int c = 0; c < n && st == FA_OK; ++c) {
        const fa_fwd_host_params &hp = ch[c].hp;
        const fa_fwd_params &p = hp.dev;
        if (cudaMemcpyAsync(const_cast<void *>(p.q), hp.q, ch[c].q_bytes, cudaMemcpyHostToDevice, cin) != cudaSuccess ||
            cudaMemcpyAsync(const_cast<void *>(p.k), hp.k, ch[c].kv_bytes, cudaMemcpyHostToDevice, cin) != cudaSuccess ||
            cudaMemcpyAsync(const_cast<void *>(p.v), hp.v, ch[c].kv_bytes, cudaMemcpyHostToDevice, cin) != cudaSuccess ||
            (hp.k_len && cudaMemcpyAsync(const_cast<int32_t *>(p.k_len), hp.k_len, sizeof(int32_t) * p.B,
                                         cudaMemcpyHostToDevice, cin) != cudaSuccess) ||
            cudaEventRecord(ev[2 + 2 * c], cin) != cudaSuccess)
            st = FA_ERR_CUDA;
    }
    for (int c = 0; c < n && st == FA_OK; ++c) {
        const fa_fwd_host_params &hp = ch[c].hp;
        const fa_fwd_params &p = hp.dev;
        if (cudaStreamWaitEvent(s, ev[2 + 2 * c], 0) != cudaSuccess) { st = FA_ERR_CUDA; break; }
        if ((st = fa_fwd_ex(&p, s)) != FA_OK) break;
        if (cudaEventRecord(ev[3 + 2 * c], s) != cudaSuccess || cudaStreamWaitEvent(cout, ev[3 + 2 * c], 0) != cudaSuccess ||
            cudaMemcpyAsync(hp.o, p.o, ch[c].o_bytes, cudaMemcpyDeviceToHost, cout) != cudaSuccess ||
            cudaMemcpyAsync(hp.lse, p.lse, ch[c].lse_bytes, cudaMemcpyDeviceToHost, cout) != cudaSuccess)
            st = FA_ERR_CUDA;
    }
    // `s` waits for the copy-out stream (and, through the events, for the copy-in stream)
    if (cudaEventRecord(end, cout) != cudaSuccess || cudaStreamWaitEvent(s, end, 0) != cudaSuccess) {
        cudaStreamSynchronize(cin);
        cudaStreamSynchronize(cout);
        if (st == FA_OK) st = FA_ERR_CUDA;
    }
    if (cudaStreamSynchronize(s) != cudaSuccess && st == FA_OK) st = FA_ERR_CUDA;
    for (int i = 0; i < n_ev; ++i)
        if (ev[i]) cudaEventDestroy(ev[i]);
    return st;
}

fa_status fa_fwd_host(const fa_fwd_host_params *hp, void *stream) {
    if (!hp) return FA_ERR_INVALID_ARGUMENT;
    const fa_fwd_params *p = &hp->dev;
    fa_status st = validate(p);
    if (st != FA_OK) return st;
    const size_t rows = (size_t)p->B * p->H * p->N;
    if (rows == 0) return FA_OK;
    if (!hp->q || !hp->k || !hp->v || !hp->o || !hp->lse) return FA_ERR_INVALID_ARGUMENT;
    if ((hp->k_len == nullptr) != (p->k_len == nullptr)) return FA_ERR_INVALID_ARGUMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int dev = 0;
    DeviceInfo *di = nullptr;
    cudaStream_t cin = nullptr, cout = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        st = probe_device(&dev, &di);
        if (st == FA_OK && !di->copy_in) {
            if (cudaStreamCreateWithFlags(&di->copy_in, cudaStreamNonBlocking) != cudaSuccess ||
                cudaStreamCreateWithFlags(&di->copy_out, cudaStreamNonBlocking) != cudaSuccess)
                st = FA_ERR_CUDA;
        }
        if (st == FA_OK) {
            cin = di->copy_in;
            cout = di->copy_out;
        }
    }
    if (st != FA_OK) return st;
    HostChunk chunks[kMaxHostChunks];
    const int n = host_chunks(hp, di->num_sms, chunks);
    if (n > 1) {
        st = host_pipelined(chunks, n, s, cin, cout);
    } else {
        st = host_single(hp, s);
        if (cudaStreamSynchronize(s) != cudaSuccess && st == FA_OK) st = FA_ERR_CUDA;
    }
    if (st != FA_OK) return st;
    if (p->dev_status) return fa_read_device_status(p->dev_status, stream);
    return FA_OK;
}

fa_status fa_read_device_status(const int32_t *dev_status, void *stream) {
    if (!dev_status) return FA_ERR_INVALID_ARGUMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int32_t h = 0;
    if (cudaMemcpyAsync(&h, dev_status, sizeof h, cudaMemcpyDeviceToHost, s) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_CUDA;
    if (h != FA_OK && h != FA_ERR_DEVICE_TIMEOUT && h != FA_ERR_SCHED_BUSY) return FA_ERR_CUDA;
    return (fa_status)h;
}

const char *fa_status_string(fa_status s) {
    switch (s) {
        case FA_OK: return "FA_OK";
        case FA_ERR_INVALID_ARGUMENT: return "FA_ERR_INVALID_ARGUMENT";
        case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED";
        case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
        case FA_ERR_CUDA: return "FA_ERR_CUDA";
        case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT";
        case FA_ERR_WORKSPACE_LIMIT: return "FA_ERR_WORKSPACE_LIMIT";
        case FA_ERR_SCHED_BUSY: return "FA_ERR_SCHED_BUSY";
    }
    return "FA_ERR_UNKNOWN";
}

int fa_version(void) { return kVersion; }

int fa_testhook_sched_next_slot(void) {
    return (int)(g_sched_next.load(std::memory_order_relaxed) % kSchedSlots);
}

fa_status fa_testhook_sched_slot(int slot, const uint32_t *set4, uint32_t *get4) {
    if (slot < 0 || slot >= kSchedSlots) return FA_ERR_INVALID_ARGUMENT;
    int dev = 0;
    DeviceInfo *di = nullptr;
    fa_status st;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        st = probe_device(&dev, &di);
    }
    if (st != FA_OK) return st;
    uint32_t *w = di->sched + kSchedWords * slot;
    if (set4 && cudaMemcpy(w, set4, kSchedWords * sizeof(uint32_t), cudaMemcpyHostToDevice) != cudaSuccess)
        return FA_ERR_CUDA;
    if (get4 && cudaMemcpy(get4, w, kSchedWords * sizeof(uint32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
        return FA_ERR_CUDA;
    return FA_OK;
}

}  // extern "C"
