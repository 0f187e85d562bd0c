// fa_api.cu -- the C ABI of libfa_sm100.so (declared in include/fa.h):
// argument checks, TMA tensor-map creation, kernel launches on the caller's
// stream, and the per-device error word that bounded device waits write.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa.h"
#include "fa_bwd64_kernel.cuh"
#include "fa_bwd_kernels.cuh"
#include "fa_decode_kernel.cuh"
#include "fa_fwd1_kernel.cuh"
#include "fa_fwd64_kernel.cuh"
#include "fa_fwd_kernel.cuh"
#include "fa_merge_kernels.cuh"

// Set (bitwise OR) by a kernel whose pipeline wait ran out; one per device.
__device__ unsigned int g_fa_error_word;
// Where the wait-timeout self-test kernel reports how its wait ended.
__device__ int g_fa_probe_result;

namespace {

constexpr int kMaxDevices = 64;

// One CTA waits, through the kernels' bounded wait, on an mbarrier that
// nothing ever arrives on; the wait runs out after `limit_ns` and records
// the timeout in the device error word exactly as a stalled pipeline would.
__global__ void fa_wait_timeout_probe_kernel(unsigned int* err, unsigned long long limit_ns,
                                             int* completed) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        fa::mbar_init(&bar, 1);
        abort_flag = 0;
        fa::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const fa::AbortState st{&abort_flag, err};
        const bool ok = fa::mbar_wait(&bar, 0, st, limit_ns);
        *completed = ok ? 1 : 2;
    }
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

struct DeviceState {
    std::once_flag once;
    bool ok = false;
    unsigned int* err_word = nullptr;
    int sm_count = 0;
    int dec_occ[2][3] = {};  // resident decode CTAs per SM: [d = 64, 128][QG = 1, 2, 4]
};
DeviceState g_dev[kMaxDevices];

bool load_encode() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

// Opts the kernel into `bytes` of dynamic shared memory and checks that the
// registers it is launched with cover its warpgroups' setmaxnreg split (an
// increase beyond the launch allocation would never be granted).
template <class K>
bool prepare_kernel(K kernel, int bytes, int threads, int reg_budget) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
        return false;
    cudaFuncAttributes attr{};
    if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) return false;
    return attr.numRegs * threads >= reg_budget;
}

template <int D, int QG>
bool prepare_decode_one(int* occ) {
    using T = fa::DecTraits<D>;
    if (cudaFuncSetAttribute(fa::fa_decode_kernel<D, QG>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             T::SMEM_BYTES) != cudaSuccess)
        return false;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, fa::fa_decode_kernel<D, QG>,
                                                         T::THREADS, T::SMEM_BYTES) ==
               cudaSuccess &&
           *occ >= 1;
}

template <int D>
bool prepare_decode(int (&occ)[3]) {
    return prepare_decode_one<D, 1>(&occ[0]) && prepare_decode_one<D, 2>(&occ[1]) &&
           prepare_decode_one<D, 4>(&occ[2]);
}

template <int D>
bool prepare_fwd_bias() {
    using T = fa::FwdTraits<D, false, true>;
    return prepare_kernel(fa::fa_fwd_kernel<D, false, false, true>, T::SMEM_BYTES,
                          T::NUM_THREADS, T::REG_BUDGET) &&
           prepare_kernel(fa::fa_fwd_kernel<D, true, false, true>, T::SMEM_BYTES, T::NUM_THREADS,
                          T::REG_BUDGET);
}

// One-time per-device set-up: architecture check, error-word address, and
// the shared-memory opt-in of every kernel.  Returns FA_OK or an error.
fa_status device_setup(int* dev_out, unsigned int** err_out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
    DeviceState& s = g_dev[dev];
    std::call_once(s.once, [&] {
        int major = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) !=
                cudaSuccess ||
            major != 10)
            return;
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fa_error_word) != cudaSuccess) return;
        s.err_word = static_cast<unsigned int*>(p);
        bool ok = true;
        ok &= prepare_kernel(fa::fa_fwd_kernel<64, false>, fa::FwdTraits<64>::SMEM_BYTES,
                             fa::FwdTraits<64>::NUM_THREADS, fa::FwdTraits<64>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_fwd_kernel<64, true>, fa::FwdTraits<64>::SMEM_BYTES,
                             fa::FwdTraits<64>::NUM_THREADS, fa::FwdTraits<64>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_fwd_kernel<128, false>, fa::FwdTraits<128>::SMEM_BYTES,
                             fa::FwdTraits<128>::NUM_THREADS, fa::FwdTraits<128>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_fwd_kernel<128, true>, fa::FwdTraits<128>::SMEM_BYTES,
                             fa::FwdTraits<128>::NUM_THREADS, fa::FwdTraits<128>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_bwd_main_kernel<64, false>, fa::BwdTraits<64>::SMEM_BYTES,
                             fa::BwdTraits<64>::NUM_THREADS, fa::BwdTraits<64>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_bwd_main_kernel<64, true>, fa::BwdTraits<64>::SMEM_BYTES,
                             fa::BwdTraits<64>::NUM_THREADS, fa::BwdTraits<64>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_bwd_main_kernel<128, false>, fa::BwdTraits<128>::SMEM_BYTES,
                             fa::BwdTraits<128>::NUM_THREADS, fa::BwdTraits<128>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_bwd_main_kernel<128, true>, fa::BwdTraits<128>::SMEM_BYTES,
                             fa::BwdTraits<128>::NUM_THREADS, fa::BwdTraits<128>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_fwd64_kernel<false>, fa::Fwd64Traits::SMEM_BYTES,
                             fa::Fwd64Traits::NUM_THREADS, fa::Fwd64Traits::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_fwd64_kernel<true>, fa::Fwd64Traits::SMEM_BYTES,
                             fa::Fwd64Traits::NUM_THREADS, fa::Fwd64Traits::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_bwd_main64_kernel<false>, fa::Bwd64Traits::SMEM_BYTES,
                             fa::Bwd64Traits::NUM_THREADS, fa::Bwd64Traits::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_bwd_main64_kernel<true>, fa::Bwd64Traits::SMEM_BYTES,
                             fa::Bwd64Traits::NUM_THREADS, fa::Bwd64Traits::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_fwd_kernel<128, false, true>,
                             fa::FwdTraits<128, true>::SMEM_BYTES,
                             fa::FwdTraits<128, true>::NUM_THREADS,
                             fa::FwdTraits<128, true>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_fwd_kernel<128, true, true>,
                             fa::FwdTraits<128, true>::SMEM_BYTES,
                             fa::FwdTraits<128, true>::NUM_THREADS,
                             fa::FwdTraits<128, true>::REG_BUDGET);
        ok &= prepare_fwd_bias<64>() && prepare_fwd_bias<128>();
        ok &= prepare_kernel(fa::fa_fwd1_kernel<64, false>, fa::Fwd1Traits<64>::SMEM_BYTES,
                             fa::Fwd1Traits<64>::NUM_THREADS, fa::Fwd1Traits<64>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_fwd1_kernel<64, true>, fa::Fwd1Traits<64>::SMEM_BYTES,
                             fa::Fwd1Traits<64>::NUM_THREADS, fa::Fwd1Traits<64>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_fwd1_kernel<128, false>, fa::Fwd1Traits<128>::SMEM_BYTES,
                             fa::Fwd1Traits<128>::NUM_THREADS, fa::Fwd1Traits<128>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_fwd1_kernel<128, true>, fa::Fwd1Traits<128>::SMEM_BYTES,
                             fa::Fwd1Traits<128>::NUM_THREADS, fa::Fwd1Traits<128>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_fwd_kernel<128, false, true, false, true>,
                             fa::FwdTraits<128, true, false, true>::SMEM_BYTES,
                             fa::FwdTraits<128, true, false, true>::NUM_THREADS,
                             fa::FwdTraits<128, true, false, true>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_fwd_kernel<128, true, true, false, true>,
                             fa::FwdTraits<128, true, false, true>::SMEM_BYTES,
                             fa::FwdTraits<128, true, false, true>::NUM_THREADS,
                             fa::FwdTraits<128, true, false, true>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_bwd_main_kernel<64, false, true>,
                             fa::BwdTraits<64>::SMEM_BYTES, fa::BwdTraits<64>::NUM_THREADS,
                             fa::BwdTraits<64>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_bwd_main_kernel<64, true, true>,
                             fa::BwdTraits<64>::SMEM_BYTES, fa::BwdTraits<64>::NUM_THREADS,
                             fa::BwdTraits<64>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_bwd_main_kernel<128, false, true>,
                             fa::BwdTraits<128>::SMEM_BYTES, fa::BwdTraits<128>::NUM_THREADS,
                             fa::BwdTraits<128>::REG_BUDGET);
        ok &= prepare_kernel(fa::fa_bwd_main_kernel<128, true, true>,
                             fa::BwdTraits<128>::SMEM_BYTES, fa::BwdTraits<128>::NUM_THREADS,
                             fa::BwdTraits<128>::REG_BUDGET);
        ok &= cudaDeviceGetAttribute(&s.sm_count, cudaDevAttrMultiProcessorCount, dev) ==
              cudaSuccess;
        ok &= prepare_decode<64>(s.dec_occ[0]);
        ok &= prepare_decode<128>(s.dec_occ[1]);
        s.ok = ok;
    });
    if (!s.ok) {
        int major = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaGetLastError();
        return major == 10 ? FA_ERR_CUDA : FA_ERR_UNSUPPORTED;
    }
    *dev_out = dev;
    *err_out = s.err_word;
    return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status check_sizes(int B, int H, int N, int d, float scale) {
    if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
    if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    const long long bh = static_cast<long long>(B) * H;
    // TMA coordinates and row indices are 32-bit; keep every index in range.
    if (bh > (1ll << 24) || N > (1 << 30) || bh * ((N + 255) / 256) > 0x7fffffffll)
        return FA_ERR_INVALID_ARG;
    return FA_OK;
}

// 3-D view [BH][rows][cols] of a row-major tensor, 128-byte swizzled boxes of
// {box_cols, box_rows, 1}.
bool encode_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
               int cols, long long rows, long long bh, int box_cols, int box_rows) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(bh)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * elem_bytes,
                             static_cast<cuuint64_t>(rows) * cols * elem_bytes};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return g_encode(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_bf16(CUtensorMap* map, const void* base, int d, int N, long long bh, int box_rows) {
    return encode_3d(map, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N, bh, 64, box_rows);
}

// mb: the bias tensor map (BIAS); other variants get any map, unused.
template <int D, bool CAUSAL, bool QK8 = false, bool BIAS = false, bool PV8 = false>
cudaError_t launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const CUtensorMap& mo, const CUtensorMap& mb, const fa::FwdParams& prm,
                       long long bh, cudaStream_t stream) {
    using T = fa::FwdTraits<D, QK8, BIAS, PV8>;
    const long long grid = bh * prm.n_qpairs;
    fa::fa_fwd_kernel<D, CAUSAL, QK8, BIAS, PV8><<<static_cast<unsigned>(grid), T::NUM_THREADS,
                                                   T::SMEM_BYTES, stream>>>(mq, mk, mv, mo, mb,
                                                                            prm);
    return cudaGetLastError();
}

// Forward kernel choice, from same-box measurements (16k tokens per batch,
// forward TFLOP/s):
//  * d = 128, N <= 512: one query tile at a time per CTA, two persistent
//    CTAs per SM (fa_fwd1_kernel), which hides the fixed cost around each
//    tile (+9% over fa_fwd_kernel); from N = 1024 on it loses up to 19%.
//  * d = 64, N <= 2048: two tiles per CTA with 64-key blocks and two CTAs
//    per SM (fa_fwd64_kernel): +24% at N = 512, +10% at N = 1024, +1-5% at
//    N = 2048 over fa_fwd_kernel, and level with or ahead of the one-tile
//    kernel; from N = 4096 on it loses 0-7%.
//  * otherwise fa_fwd_kernel: two tiles per CTA sharing every 128-key block.
// FA_FWD1_MAX_N overrides the one-tile threshold at both head dims (0:
// never) for experiments.
#ifndef FA_FWD1_MAX_N
#define FA_FWD1_MAX_N -1
#endif

// FA_FWD1_CTAS_PER_SM=0 at build time launches one CTA per tile instead of
// the persistent grid, for comparisons.
#ifndef FA_FWD1_CTAS_PER_SM
#define FA_FWD1_CTAS_PER_SM 2
#endif

bool use_fwd1(int N, int d) {
    if (FA_FWD1_MAX_N >= 0) return N <= FA_FWD1_MAX_N;
    return d == 128 && N <= 512;
}

template <int D, bool CAUSAL>
cudaError_t launch_fwd1(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const CUtensorMap& mo, const fa::FwdParams& prm, long long bh,
                        int sm_count, cudaStream_t stream) {
    using T = fa::Fwd1Traits<D>;
    // Persistent: at most two CTAs per SM (the occupancy the kernel is built
    // for), each walking every grid-th tile.
    const long long tiles = bh * ((prm.N + T::BM - 1) / T::BM);
    const long long cap = FA_FWD1_CTAS_PER_SM > 0 ? 2LL * std::max(1, sm_count) : tiles;
    const long long grid = std::min(tiles, cap);
    fa::fa_fwd1_kernel<D, CAUSAL><<<static_cast<unsigned>(grid), T::NUM_THREADS, T::SMEM_BYTES,
                                    stream>>>(mq, mk, mv, mo, prm);
    return cudaGetLastError();
}

// FA_FWD64X2=0 at build time leaves d = 64 to fa_fwd_kernel (and the
// one-tile kernel under FA_FWD1_MAX_N), for comparisons.
#ifndef FA_FWD64X2
#define FA_FWD64X2 1
#endif

bool use_fwd64(int N, int d) { return FA_FWD64X2 && FA_FWD1_MAX_N < 0 && d == 64 && N <= 2048; }

template <bool CAUSAL>
cudaError_t launch_fwd64(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& mo, const fa::FwdParams& prm, long long bh,
                         cudaStream_t stream) {
    using T = fa::Fwd64Traits;
    const long long grid = bh * prm.n_qpairs;
    fa::fa_fwd64_kernel<CAUSAL><<<static_cast<unsigned>(grid), T::NUM_THREADS, T::SMEM_BYTES,
                                  stream>>>(mq, mk, mv, mo, prm);
    return cudaGetLastError();
}

fa::FwdParams fwd_params(float* lse, unsigned int* err, int N, long long bh, int H, float sl2) {
    fa::FwdParams prm;
    prm.lse = lse;
    prm.err = err;
    prm.N = N;
    prm.n_qpairs = (N + 255) / 256;
    prm.bh_count = static_cast<int>(bh);
    prm.scale_log2 = sl2;
    prm.H = H;
    prm.bias_batch = 0;
    prm.bias_heads = 0;
    prm.strict = 0;
    prm.o_scale = 1.0f;
    return prm;
}

}  // namespace

extern "C" {

const char* fa_strerror(fa_status s) {
    switch (s) {
        case FA_OK: return "FA_OK";
        case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid argument";
        case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: unsupported head dim or device";
        case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED: pointer not 16-byte aligned";
        case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA call failed";
        case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: device pipeline wait ran out";
    }
    return "unknown fa_status";
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, int causal, float scale, void* stream) {
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    fa_status st = check_sizes(B, H, N, d, scale);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_MISALIGNED;
    if (causal < 0 || causal > 2) return FA_ERR_INVALID_ARG;
    int dev;
    unsigned int* err;
    if ((st = device_setup(&dev, &err)) != FA_OK) return st;
    if (!load_encode()) return FA_ERR_CUDA;

    const long long bh = static_cast<long long>(B) * H;
    CUtensorMap mq, mk, mv, mo;
    if (!encode_bf16(&mq, q, d, N, bh, 128) || !encode_bf16(&mk, k, d, N, bh, 128) ||
        !encode_bf16(&mv, v, d, N, bh, 128) || !encode_bf16(&mo, o, d, N, bh, 32))
        return FA_ERR_CUDA;
    fa::FwdParams prm = fwd_params(lse, err, N, bh, H, scale * 1.4426950408889634f);
    prm.strict = causal == 2;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (use_fwd64(N, d)) {
        CUtensorMap mk64, mv64;  // 64-key boxes
        if (!encode_bf16(&mk64, k, d, N, bh, 64) || !encode_bf16(&mv64, v, d, N, bh, 64))
            return FA_ERR_CUDA;
        e = causal ? launch_fwd64<true>(mq, mk64, mv64, mo, prm, bh, s)
                   : launch_fwd64<false>(mq, mk64, mv64, mo, prm, bh, s);
        return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
    }
    if (use_fwd1(N, d)) {
        if (d == 64)
            e = causal ? launch_fwd1<64, true>(mq, mk, mv, mo, prm, bh, g_dev[dev].sm_count, s)
                       : launch_fwd1<64, false>(mq, mk, mv, mo, prm, bh, g_dev[dev].sm_count, s);
        else
            e = causal ? launch_fwd1<128, true>(mq, mk, mv, mo, prm, bh, g_dev[dev].sm_count, s)
                       : launch_fwd1<128, false>(mq, mk, mv, mo, prm, bh, g_dev[dev].sm_count, s);
        return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
    }
    if (d == 64)
        e = causal ? launch_fwd<64, true>(mq, mk, mv, mo, mo, prm, bh, s)
                   : launch_fwd<64, false>(mq, mk, mv, mo, mo, prm, bh, s);
    else
        e = causal ? launch_fwd<128, true>(mq, mk, mv, mo, mo, prm, bh, s)
                   : launch_fwd<128, false>(mq, mk, mv, mo, mo, prm, bh, s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_fwd_qk8(const void* q, const void* k, const void* v, float q_descale,
                     float k_descale, void* o, float* lse, int B, int H, int N, int d,
                     int causal, float scale, void* stream) {
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    fa_status st = check_sizes(B, H, N, d, scale);
    if (st != FA_OK) return st;
    if (d != 128) return FA_ERR_UNSUPPORTED;
    if (!(std::isfinite(q_descale) && q_descale > 0.f && std::isfinite(k_descale) &&
          k_descale > 0.f))
        return FA_ERR_INVALID_ARG;
    const float sl2 = scale * q_descale * k_descale * 1.4426950408889634f;
    if (!(std::isfinite(sl2) && sl2 > 0.f)) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_MISALIGNED;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    int dev;
    unsigned int* err;
    if ((st = device_setup(&dev, &err)) != FA_OK) return st;
    if (!load_encode()) return FA_ERR_CUDA;
    const long long bh = static_cast<long long>(B) * H;
    CUtensorMap mq, mk, mv, mo;
    if (!encode_3d(&mq, q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, N, bh, 128, 128) ||
        !encode_3d(&mk, k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, N, bh, 128, 128) ||
        !encode_bf16(&mv, v, d, N, bh, 128) || !encode_bf16(&mo, o, d, N, bh, 32))
        return FA_ERR_CUDA;
    const fa::FwdParams prm = fwd_params(lse, err, N, bh, H, sl2);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e = causal ? launch_fwd<128, true, true>(mq, mk, mv, mo, mo, prm, bh, s)
                                 : launch_fwd<128, false, true>(mq, mk, mv, mo, mo, prm, bh, s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, float q_descale,
                     float k_descale, float v_descale, void* o, float* lse, int B, int H, int N,
                     int d, int causal, float scale, void* stream) {
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    fa_status st = check_sizes(B, H, N, d, scale);
    if (st != FA_OK) return st;
    if (d != 128) return FA_ERR_UNSUPPORTED;
    if (!(std::isfinite(q_descale) && q_descale > 0.f && std::isfinite(k_descale) &&
          k_descale > 0.f && std::isfinite(v_descale) && v_descale > 0.f))
        return FA_ERR_INVALID_ARG;
    const float sl2 = scale * q_descale * k_descale * 1.4426950408889634f;
    if (!(std::isfinite(sl2) && sl2 > 0.f)) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_MISALIGNED;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    int dev;
    unsigned int* err;
    if ((st = device_setup(&dev, &err)) != FA_OK) return st;
    if (!load_encode()) return FA_ERR_CUDA;
    const long long bh = static_cast<long long>(B) * H;
    CUtensorMap mq, mk, mv, mo;
    if (!encode_3d(&mq, q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, N, bh, 128, 128) ||
        !encode_3d(&mk, k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, N, bh, 128, 128) ||
        !encode_3d(&mv, v, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, N, bh, 128, 128) ||
        !encode_bf16(&mo, o, d, N, bh, 32))
        return FA_ERR_CUDA;
    fa::FwdParams prm = fwd_params(lse, err, N, bh, H, sl2);
    // O = v_descale * sum(w V8) / sum(w), with w the e4m3 weights scaled by
    // 2^PV8_P_SHIFT (the shift cancels in the ratio).
    prm.o_scale = v_descale;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e =
        causal ? launch_fwd<128, true, true, false, true>(mq, mk, mv, mo, mo, prm, bh, s)
               : launch_fwd<128, false, true, false, true>(mq, mk, mv, mo, mo, prm, bh, s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_fwd_bias(const void* q, const void* k, const void* v, const void* bias, void* o,
                      float* lse, int B, int H, int N, int d, int bias_batch, int bias_heads,
                      int causal, float scale, void* stream) {
    if (!q || !k || !v || !bias || !o || !lse) return FA_ERR_INVALID_ARG;
    fa_status st = check_sizes(B, H, N, d, scale);
    if (st != FA_OK) return st;
    if ((bias_batch != 0 && bias_batch != 1) || (bias_heads != 0 && bias_heads != 1) ||
        (causal != 0 && causal != 1))
        return FA_ERR_INVALID_ARG;
    if (N % 8 != 0) return FA_ERR_UNSUPPORTED;  // bias rows must be 16-byte multiples
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(bias) || !aligned16(o) ||
        !aligned16(lse))
        return FA_ERR_MISALIGNED;
    int dev;
    unsigned int* err;
    if ((st = device_setup(&dev, &err)) != FA_OK) return st;
    if (!load_encode()) return FA_ERR_CUDA;
    const long long bh = static_cast<long long>(B) * H;
    const long long nb = static_cast<long long>(bias_batch ? B : 1) * (bias_heads ? H : 1);
    CUtensorMap mq, mk, mv, mo, mb;
    if (!encode_bf16(&mq, q, d, N, bh, 128) || !encode_bf16(&mk, k, d, N, bh, 128) ||
        !encode_bf16(&mv, v, d, N, bh, 128) || !encode_bf16(&mo, o, d, N, bh, 32) ||
        !encode_3d(&mb, bias, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, N, nb, 64, 128))
        return FA_ERR_CUDA;
    fa::FwdParams prm = fwd_params(lse, err, N, bh, H, scale * 1.4426950408889634f);
    prm.bias_batch = bias_batch;
    prm.bias_heads = bias_heads;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (d == 64)
        e = causal ? launch_fwd<64, true, false, true>(mq, mk, mv, mo, mb, prm, bh, s)
                   : launch_fwd<64, false, false, true>(mq, mk, mv, mo, mb, prm, bh, s);
    else
        e = causal ? launch_fwd<128, true, false, true>(mq, mk, mv, mo, mb, prm, bh, s)
                   : launch_fwd<128, false, false, true>(mq, mk, mv, mo, mb, prm, bh, s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
    if (check_sizes(B, H, N, d, 1.0f) != FA_OK) return 0;
    return fa::bwd_workspace_bytes(static_cast<long long>(B) * H, N, d);
}

}  // extern "C"

namespace {

// Checks shared by the backward stages; on success fills the workspace view.
fa_status bwd_common(int B, int H, int N, int d, float scale, void* workspace,
                     size_t workspace_bytes, fa::BwdWorkspace* ws, int* dev,
                     unsigned int** err) {
    if (!workspace) return FA_ERR_INVALID_ARG;
    fa_status st = check_sizes(B, H, N, d, scale);
    if (st != FA_OK) return st;
    const long long bh = static_cast<long long>(B) * H;
    if (workspace_bytes < fa::bwd_workspace_bytes(bh, N, d)) return FA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_MISALIGNED;
    *ws = fa::bwd_workspace_layout(workspace, bh, N, d);
    return FA_OK;
}

fa_status bwd_pre_impl(const void* o, const float* lse, const void* dO, int B, int H, int N,
                       int d, void* workspace, size_t workspace_bytes, void* stream) {
    if (!o || !lse || !dO) return FA_ERR_INVALID_ARG;
    fa::BwdWorkspace ws;
    int dev;
    unsigned int* err;
    fa_status st = bwd_common(B, H, N, d, 1.0f, workspace, workspace_bytes, &ws, &dev, &err);
    if (st != FA_OK) return st;
    if (!aligned16(o) || !aligned16(lse) || !aligned16(dO)) return FA_ERR_MISALIGNED;
    if ((st = device_setup(&dev, &err)) != FA_OK) return st;
    const int bh = B * H;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e = d == 64 ? fa::launch_bwd_pre<64>(o, lse, dO, bh, N, ws, s)
                                  : fa::launch_bwd_pre<128>(o, lse, dO, bh, N, ws, s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// The backward main stage at d = 64 without a bias runs two CTAs per SM
// (fa_bwd_main64_kernel).  FA_BWD64X2=0 at build time sends it to the 64-row
// kernel with one CTA per SM instead, for comparisons.
#ifndef FA_BWD64X2
#define FA_BWD64X2 1
#endif

fa_status bwd_main_impl(const void* q, const void* k, const void* v, const void* dO, void* dk,
                        void* dv, int B, int H, int N, int d, int causal, float scale,
                        void* workspace, size_t workspace_bytes, void* stream,
                        const void* bias = nullptr, void* dbias = nullptr, int bias_batch = 0,
                        int bias_heads = 0) {
    if (!q || !k || !v || !dO || !dk || !dv) return FA_ERR_INVALID_ARG;
    if (causal < 0 || causal > (bias ? 1 : 2)) return FA_ERR_INVALID_ARG;
    fa::BwdWorkspace ws;
    int dev;
    unsigned int* err;
    fa_status st = bwd_common(B, H, N, d, scale, workspace, workspace_bytes, &ws, &dev, &err);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dk) ||
        !aligned16(dv))
        return FA_ERR_MISALIGNED;
    if ((st = device_setup(&dev, &err)) != FA_OK) return st;
    if (!load_encode()) return FA_ERR_CUDA;
    const long long bh = static_cast<long long>(B) * H;
    CUtensorMap mq, mk, mv, mdo, mdk, mdv, macc;
    if (!encode_bf16(&mq, q, d, N, bh, fa::kBwdBM) || !encode_bf16(&mk, k, d, N, bh, 128) ||
        !encode_bf16(&mv, v, d, N, bh, 128) || !encode_bf16(&mdo, dO, d, N, bh, fa::kBwdBM) ||
        !encode_bf16(&mdk, dk, d, N, bh, 32) || !encode_bf16(&mdv, dv, d, N, bh, 32) ||
        !encode_3d(&macc, ws.dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, ws.n_pad, bh, 32,
                   fa::kBwdBM))
        return FA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int ibh = static_cast<int>(bh);
    cudaError_t e;
#define FA_BWD_MAIN(DD, CC, BB)                                                            \
    fa::launch_bwd_main<DD, CC, BB>(ibh, N, scale, ws, mq, mk, mv, mdo, mdk, mdv, macc, err, s, \
                                    0, bias, dbias, H, bias_batch, bias_heads, causal == 2)
    if (FA_BWD64X2 && d == 64 && !bias) {
        e = causal ? fa::launch_bwd_main64<true>(ibh, N, scale, ws, mq, mk, mv, mdo, mdk, mdv,
                                                 macc, err, s, 0, causal == 2)
                   : fa::launch_bwd_main64<false>(ibh, N, scale, ws, mq, mk, mv, mdo, mdk, mdv,
                                                  macc, err, s, 0, 0);
    } else if (bias) {
        if (d == 64)
            e = causal ? FA_BWD_MAIN(64, true, true) : FA_BWD_MAIN(64, false, true);
        else
            e = causal ? FA_BWD_MAIN(128, true, true) : FA_BWD_MAIN(128, false, true);
    } else {
        if (d == 64)
            e = causal ? FA_BWD_MAIN(64, true, false) : FA_BWD_MAIN(64, false, false);
        else
            e = causal ? FA_BWD_MAIN(128, true, false) : FA_BWD_MAIN(128, false, false);
    }
#undef FA_BWD_MAIN
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status bwd_convert_impl(void* dq, int B, int H, int N, int d, float scale, void* workspace,
                           size_t workspace_bytes, void* stream) {
    if (!dq) return FA_ERR_INVALID_ARG;
    fa::BwdWorkspace ws;
    int dev;
    unsigned int* err;
    fa_status st = bwd_common(B, H, N, d, scale, workspace, workspace_bytes, &ws, &dev, &err);
    if (st != FA_OK) return st;
    if (!aligned16(dq)) return FA_ERR_MISALIGNED;
    if ((st = device_setup(&dev, &err)) != FA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int bh = B * H;
    const cudaError_t e = d == 64 ? fa::launch_bwd_convert<64>(dq, bh, N, scale, ws, s)
                                  : fa::launch_bwd_convert<128>(dq, bh, N, scale, ws, s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status bwd_accum_impl(const void* q, const void* k, const void* v, const void* dO,
                         float* dk_acc, float* dv_acc, int B, int H, int N, int d, int causal,
                         float scale, void* workspace, size_t workspace_bytes, void* stream) {
    if (!q || !k || !v || !dO || !dk_acc || !dv_acc) return FA_ERR_INVALID_ARG;
    if (causal < 0 || causal > 2) return FA_ERR_INVALID_ARG;
    const int strict = causal == 2;
    fa::BwdWorkspace ws;
    int dev;
    unsigned int* err;
    fa_status st = bwd_common(B, H, N, d, scale, workspace, workspace_bytes, &ws, &dev, &err);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dk_acc) ||
        !aligned16(dv_acc))
        return FA_ERR_MISALIGNED;
    if ((st = device_setup(&dev, &err)) != FA_OK) return st;
    if (!load_encode()) return FA_ERR_CUDA;
    const long long bh = static_cast<long long>(B) * H;
    CUtensorMap mq, mk, mv, mdo, mdk, mdv, macc;
    if (!encode_bf16(&mq, q, d, N, bh, fa::kBwdBM) || !encode_bf16(&mk, k, d, N, bh, 128) ||
        !encode_bf16(&mv, v, d, N, bh, 128) || !encode_bf16(&mdo, dO, d, N, bh, fa::kBwdBM) ||
        !encode_3d(&mdk, dk_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, N, bh, 32, 32) ||
        !encode_3d(&mdv, dv_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, N, bh, 32, 32) ||
        !encode_3d(&macc, ws.dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, ws.n_pad, bh, 32,
                   fa::kBwdBM))
        return FA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int ibh = static_cast<int>(bh);
    cudaError_t e;
#define FA_BWD_ACC(DD, CC)                                                                  \
    fa::launch_bwd_main<DD, CC>(ibh, N, scale, ws, mq, mk, mv, mdo, mdk, mdv, macc, err, s, 1, \
                                nullptr, nullptr, 1, 0, 0, strict)
    if (FA_BWD64X2 && d == 64)
        e = causal ? fa::launch_bwd_main64<true>(ibh, N, scale, ws, mq, mk, mv, mdo, mdk, mdv,
                                                 macc, err, s, 1, strict)
                   : fa::launch_bwd_main64<false>(ibh, N, scale, ws, mq, mk, mv, mdo, mdk, mdv,
                                                  macc, err, s, 1, 0);
    else if (d == 64)
        e = causal ? FA_BWD_ACC(64, true) : FA_BWD_ACC(64, false);
    else
        e = causal ? FA_BWD_ACC(128, true) : FA_BWD_ACC(128, false);
#undef FA_BWD_ACC
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

fa_status fa_bwd_main_accumulate(const void* q, const void* k, const void* v, const void* dO,
                                 float* dk_acc, float* dv_acc, int B, int H, int N, int d,
                                 int causal, float scale, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    return bwd_accum_impl(q, k, v, dO, dk_acc, dv_acc, B, H, N, d, causal, scale, workspace,
                          workspace_bytes, stream);
}

fa_status fa_lse_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                       void* o_out, long long rows, int d, int init, void* stream) {
    if (!o_acc || !lse_acc || !o_part || !lse_part || rows < 1 || (init != 0 && init != 1))
        return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (rows > (1ll << 40)) return FA_ERR_INVALID_ARG;
    if (!aligned16(o_acc) || !aligned16(o_part) || !aligned16(o_out)) return FA_ERR_MISALIGNED;
    int dev;
    unsigned int* err;
    fa_status st = device_setup(&dev, &err);
    if (st != FA_OK) return st;
    const long long threads = rows * (d / 8);
    const unsigned grid = static_cast<unsigned>((threads + 255) / 256);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const auto* op = static_cast<const __nv_bfloat16*>(o_part);
    auto* oo = static_cast<__nv_bfloat16*>(o_out);
    if (d == 64)
        fa::fa_lse_merge_kernel<64><<<grid, 256, 0, s>>>(o_acc, lse_acc, op, lse_part, oo, rows,
                                                         init);
    else
        fa::fa_lse_merge_kernel<128><<<grid, 256, 0, s>>>(o_acc, lse_acc, op, lse_part, oo, rows,
                                                          init);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_convert_f32_bf16(const float* src, void* dst, long long n, void* stream) {
    if (!src || !dst || n < 8 || n % 8 != 0 || n > (1ll << 42)) return FA_ERR_INVALID_ARG;
    if (!aligned16(src) || !aligned16(dst)) return FA_ERR_MISALIGNED;
    int dev;
    unsigned int* err;
    fa_status st = device_setup(&dev, &err);
    if (st != FA_OK) return st;
    const long long n8 = n / 8;
    fa::fa_f32_to_bf16_kernel<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0,
                                 static_cast<cudaStream_t>(stream)>>>(
        src, static_cast<__nv_bfloat16*>(dst), n8);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_bwd_preprocess(const void* o, const float* lse, const void* dO, int B, int H, int N,
                            int d, void* workspace, size_t workspace_bytes, void* stream) {
    return bwd_pre_impl(o, lse, dO, B, H, N, d, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_main(const void* q, const void* k, const void* v, const void* dO, void* dk,
                      void* dv, int B, int H, int N, int d, int causal, float scale,
                      void* workspace, size_t workspace_bytes, void* stream) {
    return bwd_main_impl(q, k, v, dO, dk, dv, B, H, N, d, causal, scale, workspace,
                         workspace_bytes, stream);
}

fa_status fa_bwd_dq_convert(void* dq, int B, int H, int N, int d, float scale, void* workspace,
                            size_t workspace_bytes, void* stream) {
    return bwd_convert_impl(dq, B, H, N, d, scale, workspace, workspace_bytes, stream);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                 int causal, float scale, void* workspace, size_t workspace_bytes,
                 void* stream) {
    // Validate everything before the first launch, so a failure enqueues nothing.
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv || !workspace)
        return FA_ERR_INVALID_ARG;
    fa_status st = check_sizes(B, H, N, d, scale);
    if (st != FA_OK) return st;
    if (causal < 0 || causal > 2) return FA_ERR_INVALID_ARG;
    if (workspace_bytes < fa::bwd_workspace_bytes(static_cast<long long>(B) * H, N, d))
        return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
        !aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return FA_ERR_MISALIGNED;
    int dev;
    unsigned int* err;
    if ((st = device_setup(&dev, &err)) != FA_OK) return st;
    if (!load_encode()) return FA_ERR_CUDA;
    if ((st = bwd_pre_impl(o, lse, dO, B, H, N, d, workspace, workspace_bytes, stream)) != FA_OK)
        return st;
    if ((st = bwd_main_impl(q, k, v, dO, dk, dv, B, H, N, d, causal, scale, workspace,
                            workspace_bytes, stream)) != FA_OK)
        return st;
    return bwd_convert_impl(dq, B, H, N, d, scale, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_bias(const void* q, const void* k, const void* v, const void* bias,
                      const void* o, const float* lse, const void* dO, void* dq, void* dk,
                      void* dv, void* dbias, int B, int H, int N, int d, int bias_batch,
                      int bias_heads, int causal, float scale, void* workspace,
                      size_t workspace_bytes, void* stream) {
    if (!q || !k || !v || !bias || !o || !lse || !dO || !dq || !dk || !dv || !workspace)
        return FA_ERR_INVALID_ARG;
    fa_status st = check_sizes(B, H, N, d, scale);
    if (st != FA_OK) return st;
    if ((bias_batch != 0 && bias_batch != 1) || (bias_heads != 0 && bias_heads != 1) ||
        (causal != 0 && causal != 1))
        return FA_ERR_INVALID_ARG;
    if (N % 8 != 0) return FA_ERR_UNSUPPORTED;
    if (workspace_bytes < fa::bwd_workspace_bytes(static_cast<long long>(B) * H, N, d))
        return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(bias) || !aligned16(o) ||
        !aligned16(lse) || !aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
        (dbias && !aligned16(dbias)) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return FA_ERR_MISALIGNED;
    int dev;
    unsigned int* err;
    if ((st = device_setup(&dev, &err)) != FA_OK) return st;
    if (!load_encode()) return FA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // With the causal mask the main kernel never visits the key blocks past
    // a query row's own block, whose gradient is zero: write those zeros.
    if (dbias && causal) {
        const long long rows = static_cast<long long>(B) * H * N;
        fa::fa_dbias_zero_upper_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(
            static_cast<__nv_bfloat16*>(dbias), N, rows);
        if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    if ((st = bwd_pre_impl(o, lse, dO, B, H, N, d, workspace, workspace_bytes, stream)) != FA_OK)
        return st;
    if ((st = bwd_main_impl(q, k, v, dO, dk, dv, B, H, N, d, causal, scale, workspace,
                            workspace_bytes, stream, bias, dbias, bias_batch, bias_heads)) !=
        FA_OK)
        return st;
    return bwd_convert_impl(dq, B, H, N, d, scale, workspace, workspace_bytes, stream);
}

fa_status fa_selftest_wait_timeout(unsigned int limit_us, void* stream) {
    if (limit_us == 0 || limit_us > 2000000u) return FA_ERR_INVALID_ARG;
    int dev;
    unsigned int* err;
    fa_status st = device_setup(&dev, &err);
    if (st != FA_OK) return st;
    int* completed = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&completed), g_fa_probe_result) !=
        cudaSuccess)
        return FA_ERR_CUDA;
    fa_wait_timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        err, 1000ull * limit_us, completed);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_get_device_error(void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_fa_error_word, sizeof(word)) != cudaSuccess)
        return FA_ERR_CUDA;
    if (word != 0 && cudaMemcpyToSymbol(g_fa_error_word, &zero, sizeof(zero)) != cudaSuccess)
        return FA_ERR_CUDA;
    if (word & fa::kErrTimeout) return FA_ERR_TIMEOUT;
    return word ? FA_ERR_CUDA : FA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ decoding

namespace {

int decode_qgroup_rows(int Nq) { return Nq == 1 ? 1 : Nq == 2 ? 2 : 4; }

long long decode_max_splits(int Nk) {
    return (static_cast<long long>(Nk) + fa::kDecodeMinChunk - 1) / fa::kDecodeMinChunk;
}

fa_status decode_check(int B, int H, int Nq, int Nk, int d, float scale) {
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
    if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    const long long bh = static_cast<long long>(B) * H;
    // Grid indices (one CTA per head x split x query group) are 32-bit.
    if (bh > (1ll << 24) || Nq > (1 << 24) || Nk > (1 << 30) ||
        bh * ((Nq + 3) / 4) * decode_max_splits(Nk) > 0x7fffffffll)
        return FA_ERR_INVALID_ARG;
    return FA_OK;
}

// Cost model of the split choice, in units of the time one CTA takes to
// stream one key row.  One CTA streams at a rate set by the bytes it keeps in
// flight (its pipeline stages); HBM saturates once about kSatBytesPerSm x SMs
// bytes are in flight, i.e. with R = that / (bytes per CTA) CTAs streaming.  A
// wave of n resident CTAs over `chunk` keys therefore lasts
// chunk * max(1, n / R); each wave adds a fixed ramp (first copies, merge of
// the warp groups) and splitting adds the merge launch.
constexpr long long kSatBytesPerSm = 130 << 10;
constexpr long long kWaveOverheadKeys = 256;
constexpr long long kMergeOverheadKeys = 128;

}  // namespace

extern "C" {

fa_status fa_decode_split_plan(int B, int H, int Nq, int Nk, int d, int sm_count,
                               int ctas_per_sm, int* qgroup_rows, int* n_splits, int* chunk) {
    if (!qgroup_rows || !n_splits || !chunk || sm_count < 1 || ctas_per_sm < 1)
        return FA_ERR_INVALID_ARG;
    fa_status st = decode_check(B, H, Nq, Nk, d, 1.0f);
    if (st != FA_OK) return st;
    constexpr int BK = fa::DecTraits<64>::BK;
    static_assert(fa::DecTraits<128>::BK == BK, "one key block size for both head dims");
    const int qg = decode_qgroup_rows(Nq);
    const long long units = static_cast<long long>(B) * H * ((Nq + qg - 1) / qg);
    const long long slots = static_cast<long long>(sm_count) * ctas_per_sm;
    const long long smax = std::min<long long>(decode_max_splits(Nk), 4 * slots);
    const long long inflight = d == 128
                                   ? static_cast<long long>(fa::DecTraits<128>::BAR_OFF)
                                   : static_cast<long long>(fa::DecTraits<64>::BAR_OFF);
    const double sat = std::max(1.0, static_cast<double>(kSatBytesPerSm) * sm_count / inflight);
    // The cheapest split count under the cost model above; the smallest on
    // ties.  Splits that would leave the last one empty are skipped.
    double best_cost = -1.0;
    int best_s = 1, best_chunk = (Nk + BK - 1) / BK * BK;
    for (long long s = 1; s <= smax; ++s) {
        const long long c = ((Nk + s - 1) / s + BK - 1) / BK * BK;
        if (s > 1 && c < fa::kDecodeMinChunk) break;
        const long long s_eff = (Nk + c - 1) / c;
        if (s_eff != s) continue;
        const long long ctas = units * s;
        const long long full_waves = ctas / slots, rest = ctas % slots;
        double cost = static_cast<double>(full_waves) *
                      (c * std::max(1.0, slots / sat) + kWaveOverheadKeys);
        if (rest) cost += c * std::max(1.0, rest / sat) + kWaveOverheadKeys;
        if (s > 1) cost += kMergeOverheadKeys;
        if (best_cost < 0 || cost < best_cost * (1.0 - 1e-9)) {
            best_cost = cost;
            best_s = static_cast<int>(s);
            best_chunk = static_cast<int>(c);
        }
    }
    *qgroup_rows = qg;
    *n_splits = best_s;
    *chunk = best_chunk;
    return FA_OK;
}

size_t fa_decode_workspace_size(int B, int H, int Nq, int Nk, int d) {
    if (decode_check(B, H, Nq, Nk, d, 1.0f) != FA_OK) return 0;
    const long long smax = decode_max_splits(Nk);
    if (smax <= 1) return 0;
    return static_cast<size_t>(B) * H * Nq * smax * (d + 1) * sizeof(float);
}

}  // extern "C"

namespace {

template <int D, int QG>
cudaError_t launch_decode(const fa::DecodeParams& prm, long long bh, cudaStream_t stream) {
    using T = fa::DecTraits<D>;
    const long long grid = bh * prm.n_splits * prm.n_qgroups;
    fa::fa_decode_kernel<D, QG>
        <<<static_cast<unsigned>(grid), T::THREADS, T::SMEM_BYTES, stream>>>(prm);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || prm.n_splits == 1) return e;
    const long long rows = bh * prm.Nq;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((rows + 3) / 4));
    cfg.blockDim = dim3(128);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fa::fa_decode_combine_kernel<D>,
                              static_cast<const float*>(prm.part_o),
                              static_cast<const float*>(prm.part_lse), prm.o, prm.lse, rows,
                              prm.n_splits);
}

template <int D>
cudaError_t launch_decode_d(const fa::DecodeParams& prm, int qg, long long bh,
                            cudaStream_t stream) {
    return qg == 1   ? launch_decode<D, 1>(prm, bh, stream)
           : qg == 2 ? launch_decode<D, 2>(prm, bh, stream)
                     : launch_decode<D, 4>(prm, bh, stream);
}

}  // namespace

extern "C" {

fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int Nq, int Nk, long long kv_rows, int d, int causal,
                        float scale, void* workspace, size_t workspace_bytes, void* stream) {
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    fa_status st = decode_check(B, H, Nq, Nk, d, scale);
    if (st != FA_OK) return st;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (causal && Nk < Nq) return FA_ERR_INVALID_ARG;
    if (kv_rows < Nk || kv_rows > (1ll << 40)) return FA_ERR_INVALID_ARG;
    const size_t need = fa_decode_workspace_size(B, H, Nq, Nk, d);
    if (need > 0 && (!workspace || workspace_bytes < need)) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return FA_ERR_MISALIGNED;
    int dev;
    unsigned int* err;
    if ((st = device_setup(&dev, &err)) != FA_OK) return st;
    const DeviceState& ds = g_dev[dev];
    const int qg = decode_qgroup_rows(Nq);
    const int occ = ds.dec_occ[d == 128][qg == 1 ? 0 : qg == 2 ? 1 : 2];
    int qg_rows = 0, n_splits = 0, chunk = 0;
    if ((st = fa_decode_split_plan(B, H, Nq, Nk, d, ds.sm_count, occ, &qg_rows, &n_splits,
                                   &chunk)) != FA_OK)
        return st;
    const long long bh = static_cast<long long>(B) * H;
    fa::DecodeParams prm;
    prm.q = static_cast<const __nv_bfloat16*>(q);
    prm.k = static_cast<const __nv_bfloat16*>(k);
    prm.v = static_cast<const __nv_bfloat16*>(v);
    prm.o = static_cast<__nv_bfloat16*>(o);
    prm.lse = lse;
    prm.part_o = static_cast<float*>(workspace);
    prm.part_lse = n_splits > 1 ? prm.part_o + bh * Nq * n_splits * d : nullptr;
    prm.err = err;
    prm.kv_rows = kv_rows;
    prm.Nq = Nq;
    prm.Nk = Nk;
    prm.n_qgroups = (Nq + qg - 1) / qg;
    prm.n_splits = n_splits;
    prm.chunk = chunk;
    prm.causal = causal;
    prm.scale_log2 = scale * 1.4426950408889634f;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e = d == 64 ? launch_decode_d<64>(prm, qg, bh, s)
                                  : launch_decode_d<128>(prm, qg, bh, s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"
