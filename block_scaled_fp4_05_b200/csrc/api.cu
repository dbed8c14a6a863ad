// extern "C" entry points of libfp4 (declared in include/fp4.h): host-side
// argument checks, then kernel launches on the caller's stream.

#include <cuda_runtime.h>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include <vector>

#include "fp4_internal.h"

namespace fp4 {

cudaError_t device_info(DeviceInfo* out)
{
    static std::mutex mu;
    static DeviceInfo cache[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && cache[dev].sm_count > 0) {
        *out = cache[dev];
        return cudaSuccess;
    }
    DeviceInfo d;
    e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return e;
    if (dev < 64) cache[dev] = d;
    *out = d;
    return cudaSuccess;
}

thread_local char g_last_error[256] = "";

cudaError_t current_context(void** ctx)
{
    using GetCurrentFn = int (*)(void**);   // cuCtxGetCurrent, reached through the runtime
    static GetCurrentFn fn = []() -> GetCurrentFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<GetCurrentFn>(p);
    }();
    if (!fn) return cudaErrorNotSupported;
    *ctx = nullptr;
    return fn(ctx) == 0 ? cudaSuccess : cudaErrorInvalidResourceHandle;
}

void set_last_error(const char* what, cudaError_t e)
{
    snprintf(g_last_error, sizeof g_last_error, "%s: %s", what,
             e == cudaSuccess ? "invalid argument" : cudaGetErrorString(e));
}

}  // namespace fp4

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Formats of the GEMM and quantizer entry points.
bool valid_fmt(fp4_format f) { return f == FP4_NVFP4 || f == FP4_MXFP4 || f == FP4_P1E8; }
bool valid_quant_fmt(fp4_format f) { return valid_fmt(f); }

fp4_status from_cuda(cudaError_t e)
{
    if (e == cudaSuccess) return FP4_OK;
    if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver) return FP4_ERR_NO_DEVICE;
    return FP4_ERR_CUDA;
}

// The kernels use tcgen05 / TMA instructions of sm_100a.
fp4_status require_device(fp4::DeviceInfo* dev)
{
    cudaError_t e = fp4::device_info(dev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return from_cuda(e);
    }
    if (dev->major != 10) return FP4_ERR_NO_DEVICE;
    return FP4_OK;
}

constexpr int64_t kMaxGridY = 65535;
constexpr int64_t kMaxRows = (int64_t)1 << 31;
// Rowwise tiles (128 rows x 4 blocks) of one tensor: a batched launch puts
// the tiles of up to 8 tensors in one 1-D grid.
constexpr int64_t kMaxRowTiles = (int64_t)1 << 28;

}  // namespace

extern "C" {

int fp4_abi_version(void) { return 4; }

const char* fp4_last_error(void) { return fp4::g_last_error; }

const char* fp4_status_string(fp4_status s)
{
    switch (s) {
    case FP4_OK: return "FP4_OK";
    case FP4_ERR_INVALID_ARG: return "FP4_ERR_INVALID_ARG";
    case FP4_ERR_UNSUPPORTED_SHAPE: return "FP4_ERR_UNSUPPORTED_SHAPE";
    case FP4_ERR_MISALIGNED: return "FP4_ERR_MISALIGNED";
    case FP4_ERR_CUDA: return "FP4_ERR_CUDA";
    case FP4_ERR_TIMEOUT: return "FP4_ERR_TIMEOUT";
    case FP4_ERR_NO_DEVICE: return "FP4_ERR_NO_DEVICE";
    case FP4_ERR_WORKSPACE: return "FP4_ERR_WORKSPACE";
    }
    return "FP4_ERR_UNKNOWN";
}

size_t fp4_packed_bytes(int64_t rows, int64_t k)
{
    if (rows <= 0 || k <= 0) return 0;
    return (size_t)rows * (size_t)(k / 2);
}

size_t fp4_scale_bytes(fp4_format fmt, int64_t rows, int64_t k)
{
    if (!valid_quant_fmt(fmt) || rows <= 0 || k <= 0) return 0;
    const int64_t nsc = k / fp4::block_size(fmt);
    return (size_t)((rows + 127) / 128) * (size_t)((nsc + 3) / 4) * 512u;
}

fp4_status fp4_compute_global_scale(const void* in_bf16, int64_t rows, int64_t cols, int64_t ld,
                                    float* gs_out, fp4_stream_t stream)
{
    fp4::g_last_error[0] = 0;
    if (rows < 0 || cols < 0 || gs_out == nullptr) return FP4_ERR_INVALID_ARG;
    if (rows > 0 && cols > 0 && in_bf16 == nullptr) return FP4_ERR_INVALID_ARG;
    if (ld < cols) return FP4_ERR_INVALID_ARG;
    if (cols % 8 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (ld % 8 != 0 || !aligned16(in_bf16) || (reinterpret_cast<uintptr_t>(gs_out) & 3u))
        return FP4_ERR_MISALIGNED;
    fp4::DeviceInfo dev;
    fp4_status st = require_device(&dev);
    if (st != FP4_OK) return st;
    return from_cuda(fp4::launch_global_scale(static_cast<const uint16_t*>(in_bf16), rows, cols, ld,
                                              gs_out, nullptr, nullptr,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

fp4_status fp4_compute_global_scale_alpha(const void* in_bf16, int64_t rows, int64_t cols, int64_t ld,
                                          float* gs_out, const float* other_gs, float* alpha_out,
                                          fp4_stream_t stream)
{
    fp4::g_last_error[0] = 0;
    if (rows < 0 || cols < 0 || gs_out == nullptr || other_gs == nullptr || alpha_out == nullptr)
        return FP4_ERR_INVALID_ARG;
    if (rows > 0 && cols > 0 && in_bf16 == nullptr) return FP4_ERR_INVALID_ARG;
    if (ld < cols) return FP4_ERR_INVALID_ARG;
    if (cols % 8 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (ld % 8 != 0 || !aligned16(in_bf16) || (reinterpret_cast<uintptr_t>(gs_out) & 3u) ||
        (reinterpret_cast<uintptr_t>(other_gs) & 3u) || (reinterpret_cast<uintptr_t>(alpha_out) & 3u))
        return FP4_ERR_MISALIGNED;
    fp4::DeviceInfo dev;
    fp4_status st = require_device(&dev);
    if (st != FP4_OK) return st;
    return from_cuda(fp4::launch_global_scale(static_cast<const uint16_t*>(in_bf16), rows, cols, ld,
                                              gs_out, other_gs, alpha_out,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

fp4_status fp4_compute_global_scales_pair(const void* a_bf16, int64_t rows_a, int64_t cols_a,
                                          int64_t ld_a, const void* b_bf16, int64_t rows_b,
                                          int64_t cols_b, int64_t ld_b, float* gs_a_out,
                                          float* gs_b_out, float* alpha_out, fp4_stream_t stream)
{
    fp4::g_last_error[0] = 0;
    if (rows_a < 0 || cols_a < 0 || rows_b < 0 || cols_b < 0 || gs_a_out == nullptr || gs_b_out == nullptr)
        return FP4_ERR_INVALID_ARG;
    if ((rows_a > 0 && cols_a > 0 && a_bf16 == nullptr) || (rows_b > 0 && cols_b > 0 && b_bf16 == nullptr))
        return FP4_ERR_INVALID_ARG;
    if (ld_a < cols_a || ld_b < cols_b) return FP4_ERR_INVALID_ARG;
    if (cols_a % 8 != 0 || cols_b % 8 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (ld_a % 8 != 0 || ld_b % 8 != 0 || !aligned16(a_bf16) || !aligned16(b_bf16) ||
        (reinterpret_cast<uintptr_t>(gs_a_out) & 3u) || (reinterpret_cast<uintptr_t>(gs_b_out) & 3u) ||
        (reinterpret_cast<uintptr_t>(alpha_out) & 3u))
        return FP4_ERR_MISALIGNED;
    fp4::DeviceInfo dev;
    fp4_status st = require_device(&dev);
    if (st != FP4_OK) return st;
    return from_cuda(fp4::launch_global_scale_pair(
        static_cast<const uint16_t*>(a_bf16), rows_a, cols_a, ld_a, static_cast<const uint16_t*>(b_bf16), rows_b,
        cols_b, ld_b, gs_a_out, gs_b_out, alpha_out, reinterpret_cast<cudaStream_t>(stream)));
}

fp4_status fp4_quantize(fp4_format fmt, fp4_axis axis, const void* in_bf16, int64_t rows,
                        int64_t cols, int64_t ld, void* packed_out, void* scales_out,
                        const float* global_scale, fp4_stream_t stream)
{
    fp4::g_last_error[0] = 0;
    if (!valid_quant_fmt(fmt) || (axis != FP4_ROWWISE && axis != FP4_COLWISE)) return FP4_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols) return FP4_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return FP4_OK;
    if (!in_bf16 || !packed_out || !scales_out) return FP4_ERR_INVALID_ARG;
    if (fmt != FP4_MXFP4 && !global_scale) return FP4_ERR_INVALID_ARG;
    const int kb = fp4::block_size(fmt);
    if (axis == FP4_ROWWISE) {
        if (cols % (4 * kb) != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
        if (rows >= kMaxRows || cols >= kMaxRows || ((rows + 127) / 128) * (cols / (4 * kb)) > kMaxRowTiles)
            return FP4_ERR_UNSUPPORTED_SHAPE;
    } else {
        if (rows % (4 * kb) != 0 || cols % 8 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
        if ((cols + 127) / 128 > kMaxGridY) return FP4_ERR_UNSUPPORTED_SHAPE;
    }
    if (ld % 8 != 0 || !aligned16(in_bf16) || !aligned16(packed_out) || !aligned16(scales_out))
        return FP4_ERR_MISALIGNED;
    if (global_scale && (reinterpret_cast<uintptr_t>(global_scale) & 3u)) return FP4_ERR_MISALIGNED;
    fp4::DeviceInfo dev;
    fp4_status st = require_device(&dev);
    if (st != FP4_OK) return st;
    return from_cuda(fp4::launch_quantize(
        (int)fmt, (int)axis, static_cast<const uint16_t*>(in_bf16), rows, cols, ld,
        static_cast<uint8_t*>(packed_out), static_cast<uint8_t*>(scales_out),
        fmt != FP4_MXFP4 ? global_scale : nullptr, reinterpret_cast<cudaStream_t>(stream)));
}

fp4_status fp4_quantize_batch(fp4_format fmt, int n, const fp4_quantize_desc* descs,
                              fp4_stream_t stream)
{
    fp4::g_last_error[0] = 0;
    if (!valid_quant_fmt(fmt) || n < 0 || (n > 0 && !descs)) return FP4_ERR_INVALID_ARG;
    const int kb = fp4::block_size(fmt);
    int work = 0;
    for (int i = 0; i < n; ++i) {
        const fp4_quantize_desc& d = descs[i];
        if (d.rows < 0 || d.cols < 0 || d.ld < d.cols) return FP4_ERR_INVALID_ARG;
        if (d.rows == 0 || d.cols == 0) continue;
        ++work;
        if (!d.in_bf16 || !d.packed_out || !d.scales_out) return FP4_ERR_INVALID_ARG;
        if (fmt != FP4_MXFP4 && !d.global_scale) return FP4_ERR_INVALID_ARG;
        if (d.cols % (4 * kb) != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
        if (d.rows >= kMaxRows || d.cols >= kMaxRows || ((d.rows + 127) / 128) * (d.cols / (4 * kb)) > kMaxRowTiles)
            return FP4_ERR_UNSUPPORTED_SHAPE;
        if (d.ld % 8 != 0 || !aligned16(d.in_bf16) || !aligned16(d.packed_out) || !aligned16(d.scales_out))
            return FP4_ERR_MISALIGNED;
        if (d.global_scale && (reinterpret_cast<uintptr_t>(d.global_scale) & 3u)) return FP4_ERR_MISALIGNED;
    }
    if (work == 0) return FP4_OK;
    fp4::DeviceInfo dev;
    fp4_status st = require_device(&dev);
    if (st != FP4_OK) return st;
    fp4::RowwiseDesc local[16];
    for (int i0 = 0; i0 < n; i0 += 16) {
        const int m = n - i0 < 16 ? n - i0 : 16;
        for (int i = 0; i < m; ++i) {
            const fp4_quantize_desc& d = descs[i0 + i];
            local[i] = {static_cast<const uint16_t*>(d.in_bf16), d.rows, d.cols, d.ld,
                        static_cast<uint8_t*>(d.packed_out), static_cast<uint8_t*>(d.scales_out),
                        fmt != FP4_MXFP4 ? d.global_scale : nullptr};
        }
        st = from_cuda(fp4::launch_quantize_rowwise_batch((int)fmt, m, local,
                                                          reinterpret_cast<cudaStream_t>(stream)));
        if (st != FP4_OK) return st;
    }
    return FP4_OK;
}

fp4_status fp4_dequantize(fp4_format fmt, const void* packed, const void* scales,
                          const float* global_scale, int64_t rows, int64_t k, void* out_bf16,
                          int64_t ld, fp4_stream_t stream)
{
    fp4::g_last_error[0] = 0;
    if (!valid_quant_fmt(fmt) || rows < 0 || k < 0 || ld < k) return FP4_ERR_INVALID_ARG;
    if (rows == 0 || k == 0) return FP4_OK;
    if (!packed || !scales || !out_bf16) return FP4_ERR_INVALID_ARG;
    if (fmt != FP4_MXFP4 && !global_scale) return FP4_ERR_INVALID_ARG;
    if (k % (4 * fp4::block_size(fmt)) != 0 || rows >= kMaxRows || k >= kMaxRows)
        return FP4_ERR_UNSUPPORTED_SHAPE;
    if (ld % 8 != 0 || !aligned16(packed) || !aligned16(out_bf16)) return FP4_ERR_MISALIGNED;
    if (global_scale && (reinterpret_cast<uintptr_t>(global_scale) & 3u)) return FP4_ERR_MISALIGNED;
    fp4::DeviceInfo dev;
    fp4_status st = require_device(&dev);
    if (st != FP4_OK) return st;
    return from_cuda(fp4::launch_dequantize(
        (int)fmt, static_cast<const uint8_t*>(packed), static_cast<const uint8_t*>(scales),
        fmt != FP4_MXFP4 ? global_scale : nullptr, rows, k, static_cast<uint16_t*>(out_bf16), ld,
        reinterpret_cast<cudaStream_t>(stream)));
}

fp4_status fp4_quantize_dynamic(fp4_format fmt, const void* in_bf16, int64_t rows, int64_t cols,
                                int64_t ld, void* packed_out, void* scales_out, float* gs_out,
                                const float* other_gs, float* alpha_out, fp4_stream_t stream)
{
    fp4::g_last_error[0] = 0;
    if (fmt != FP4_NVFP4) return FP4_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols || !gs_out) return FP4_ERR_INVALID_ARG;
    if (alpha_out && !other_gs) return FP4_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (!in_bf16 || !packed_out || !scales_out) return FP4_ERR_INVALID_ARG;
    if (cols % 64 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (ld % 8 != 0 || !aligned16(in_bf16) || !aligned16(packed_out) || !aligned16(scales_out))
        return FP4_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(gs_out) & 3u) || (alpha_out && (reinterpret_cast<uintptr_t>(alpha_out) & 3u)) ||
        (other_gs && (reinterpret_cast<uintptr_t>(other_gs) & 3u)))
        return FP4_ERR_MISALIGNED;
    fp4::DeviceInfo dev;
    fp4_status st = require_device(&dev);
    if (st != FP4_OK) return st;
    return from_cuda(fp4::launch_quantize_dynamic(
        static_cast<const uint16_t*>(in_bf16), rows, cols, ld, static_cast<uint8_t*>(packed_out),
        static_cast<uint8_t*>(scales_out), gs_out, other_gs, alpha_out,
        reinterpret_cast<cudaStream_t>(stream)));
}

fp4_status fp4_alpha_from_global_scales(const float* gsA, const float* gsB, float* alpha_out,
                                        fp4_stream_t stream)
{
    fp4::g_last_error[0] = 0;
    if (!gsA || !gsB || !alpha_out) return FP4_ERR_INVALID_ARG;
    fp4::DeviceInfo dev;
    fp4_status st = require_device(&dev);
    if (st != FP4_OK) return st;
    return from_cuda(fp4::launch_alpha(gsA, gsB, alpha_out, reinterpret_cast<cudaStream_t>(stream)));
}

size_t fp4_gemm_workspace_bytes(fp4_format fmt, int64_t M, int64_t N, int64_t K)
{
    if (!valid_fmt(fmt)) return 0;
    fp4::DeviceInfo dev;
    if (fp4::device_info(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return fp4::decode_workspace_bytes(M, N, K, dev.sm_count);
}

// Checks of one GEMM problem with M, N > 0 (shared by fp4_gemm and
// fp4_gemm_grouped).
static fp4_status validate_gemm(fp4_format fmt, const void* A, const void* sA, const void* B,
                                const void* sB, int64_t M, int64_t N, int64_t K, const float* alpha,
                                const void* D, int64_t ldd)
{
    if (M < 0 || N < 0 || K < 0 || ldd < N) return FP4_ERR_INVALID_ARG;
    if (!D) return FP4_ERR_INVALID_ARG;
    const int kq = fmt == FP4_MXFP4 ? 128 : 64;   // four blocks: whole scale tiles
    if (K % kq != 0 || N % 8 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (M >= kMaxRows || N >= kMaxRows || K / 2 >= kMaxRows) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (ldd % 8 != 0 || !aligned16(D)) return FP4_ERR_MISALIGNED;
    if (K > 0) {
        if (!A || !sA || !B || !sB) return FP4_ERR_INVALID_ARG;
        if (!aligned16(A) || !aligned16(B) || !aligned16(sA) || !aligned16(sB))
            return FP4_ERR_MISALIGNED;
    }
    if (alpha && (reinterpret_cast<uintptr_t>(alpha) & 3u)) return FP4_ERR_MISALIGNED;
    return FP4_OK;
}

fp4_status fp4_gemm_grouped(fp4_format fmt, int n, const fp4_gemm_problem* problems, fp4_stream_t stream)
{
    fp4::g_last_error[0] = 0;
    if (!valid_fmt(fmt) || n < 0 || (n > 0 && !problems)) return FP4_ERR_INVALID_ARG;
    int work = 0;
    for (int i = 0; i < n; ++i) {
        const fp4_gemm_problem& q = problems[i];
        if (q.M < 0 || q.N < 0 || q.K < 0) return FP4_ERR_INVALID_ARG;
        if (q.M == 0 || q.N == 0) continue;
        const fp4_status vs = validate_gemm(fmt, q.A, q.sA, q.B, q.sB, q.M, q.N, q.K, q.alpha, q.D, q.ldd);
        if (vs != FP4_OK) return vs;
        ++work;
    }
    if (work == 0) return FP4_OK;
    fp4::DeviceInfo dev;
    fp4_status st = require_device(&dev);
    if (st != FP4_OK) return st;
    if (!fp4::tensor_map_encoder_available()) return FP4_ERR_NO_DEVICE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    std::vector<fp4::GemmArgs> args;
    args.reserve(n);
    for (int i = 0; i < n; ++i) {
        const fp4_gemm_problem& q = problems[i];
        if (q.M == 0 || q.N == 0) continue;
        if (q.K == 0) {   // D = 0
            st = from_cuda(cudaMemset2DAsync(q.D, (size_t)q.ldd * 2, 0, (size_t)q.N * 2, (size_t)q.M, s));
            if (st != FP4_OK) return st;
            continue;
        }
        fp4::GemmArgs a;
        a.fmt = (int)fmt;
        a.A = static_cast<const uint8_t*>(q.A);
        a.sA = static_cast<const uint8_t*>(q.sA);
        a.B = static_cast<const uint8_t*>(q.B);
        a.sB = static_cast<const uint8_t*>(q.sB);
        a.M = q.M;
        a.N = q.N;
        a.K = q.K;
        a.alpha = q.alpha;
        a.D = static_cast<uint16_t*>(q.D);
        a.ldd = q.ldd;
        a.ws = nullptr;
        a.ws_bytes = 0;
        a.b_static = false;
        args.push_back(a);
    }
    return from_cuda(fp4::launch_gemm_grouped((int)args.size(), args.data(), dev, s));
}

fp4_status fp4_gemm_with_kernel(fp4_format fmt, const void* A, const void* sA, const void* B,
                                const void* sB, int64_t M, int64_t N, int64_t K,
                                const float* alpha, void* D, int64_t ldd, void* workspace,
                                size_t ws_bytes, fp4_gemm_kernel kernel, fp4_stream_t stream)
{
    fp4::g_last_error[0] = 0;
    if (!valid_fmt(fmt)) return FP4_ERR_INVALID_ARG;
    const int flags = (int)kernel & ~0xFF;
    kernel = (fp4_gemm_kernel)((int)kernel & 0xFF);
    if (kernel != FP4_GEMM_AUTO && kernel != FP4_GEMM_PREFILL && kernel != FP4_GEMM_DECODE)
        return FP4_ERR_INVALID_ARG;
    if (flags & ~(int)FP4_GEMM_B_STATIC) return FP4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) {
        if (M < 0 || N < 0 || K < 0 || ldd < N) return FP4_ERR_INVALID_ARG;
        return FP4_OK;
    }
    const fp4_status vs = validate_gemm(fmt, A, sA, B, sB, M, N, K, alpha, D, ldd);
    if (vs != FP4_OK) return vs;
    fp4::DeviceInfo dev;
    fp4_status st = require_device(&dev);
    if (st != FP4_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (K == 0) {
        return from_cuda(cudaMemset2DAsync(D, (size_t)ldd * 2, 0, (size_t)N * 2, (size_t)M, s));
    }
    if (!fp4::tensor_map_encoder_available()) return FP4_ERR_NO_DEVICE;

    const size_t need = fp4::decode_workspace_bytes(M, N, K, dev.sm_count);
    bool decode = false;
    if (kernel == FP4_GEMM_DECODE) {
        if (M > 16 || need == 0) return FP4_ERR_UNSUPPORTED_SHAPE;   // need == 0: N beyond the counters
        if (!workspace || ws_bytes < need) return FP4_ERR_INVALID_ARG;
        if (!aligned16(workspace)) return FP4_ERR_MISALIGNED;
        decode = true;
    } else if (kernel == FP4_GEMM_AUTO) {
        decode = M <= 16 && need > 0 && workspace && ws_bytes >= need && aligned16(workspace);
    }
    fp4::GemmArgs a;
    a.fmt = (int)fmt;
    a.A = static_cast<const uint8_t*>(A);
    a.sA = static_cast<const uint8_t*>(sA);
    a.B = static_cast<const uint8_t*>(B);
    a.sB = static_cast<const uint8_t*>(sB);
    a.M = M;
    a.N = N;
    a.K = K;
    a.alpha = alpha;
    a.D = static_cast<uint16_t*>(D);
    a.ldd = ldd;
    a.ws = workspace;
    a.ws_bytes = ws_bytes;
    a.b_static = (flags & FP4_GEMM_B_STATIC) != 0;
    const cudaError_t e = decode ? fp4::launch_gemm_decode(a, dev, s) : fp4::launch_gemm_prefill(a, dev, s);
    return from_cuda(e);
}

fp4_status fp4_gemm(fp4_format fmt, const void* A, const void* sA, const void* B, const void* sB,
                    int64_t M, int64_t N, int64_t K, const float* alpha, void* D, int64_t ldd,
                    void* workspace, size_t ws_bytes, fp4_stream_t stream)
{
    return fp4_gemm_with_kernel(fmt, A, sA, B, sB, M, N, K, alpha, D, ldd, workspace, ws_bytes,
                                FP4_GEMM_AUTO, stream);
}

fp4_status fp4_gemm_decode_dynamic(const void* act_bf16, int64_t lda, const void* W, const void* sW,
                                   const float* gsW, int64_t M, int64_t N, int64_t K, void* D,
                                   int64_t ldd, float* gsA_out, float* alpha_out, void* workspace,
                                   size_t ws_bytes, fp4_stream_t stream)
{
    fp4::g_last_error[0] = 0;
    if (M < 0 || N < 0 || K < 0 || !gsW || !gsA_out || !alpha_out) return FP4_ERR_INVALID_ARG;
    if (M > 16) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) {
        if (ldd < N) return FP4_ERR_INVALID_ARG;
        return FP4_OK;
    }
    if (K == 0 || K % 64 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (!act_bf16 || lda < K) return FP4_ERR_INVALID_ARG;
    if (lda % 8 != 0 || !aligned16(act_bf16) || (reinterpret_cast<uintptr_t>(gsW) & 3u) ||
        (reinterpret_cast<uintptr_t>(gsA_out) & 3u) || (reinterpret_cast<uintptr_t>(alpha_out) & 3u))
        return FP4_ERR_MISALIGNED;
    // the weight side as in fp4_gemm (the packed activation arguments are unused)
    const fp4_status vs = validate_gemm(FP4_NVFP4, W, sW, W, sW, M, N, K, alpha_out, D, ldd);
    if (vs != FP4_OK) return vs;
    fp4::DeviceInfo dev;
    fp4_status st = require_device(&dev);
    if (st != FP4_OK) return st;
    if (!fp4::tensor_map_encoder_available()) return FP4_ERR_NO_DEVICE;
    const size_t need = fp4::decode_workspace_bytes(M, N, K, dev.sm_count);
    if (need == 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (!workspace || ws_bytes < need) return FP4_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return FP4_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // S_global of the activation and alpha in one launch, then the GEMM
    cudaError_t e = fp4::launch_global_scale(static_cast<const uint16_t*>(act_bf16), M, K, lda, gsA_out,
                                             gsW, alpha_out, s);
    if (e != cudaSuccess) {
        fp4::set_last_error("activation S_global launch", e);
        return from_cuda(e);
    }
    fp4::GemmArgs a;
    a.fmt = fp4::kNv;
    a.A = nullptr;
    a.sA = nullptr;
    a.B = static_cast<const uint8_t*>(W);
    a.sB = static_cast<const uint8_t*>(sW);
    a.M = M;
    a.N = N;
    a.K = K;
    a.alpha = alpha_out;
    a.D = static_cast<uint16_t*>(D);
    a.ldd = ldd;
    a.ws = workspace;
    a.ws_bytes = ws_bytes;
    a.b_static = true;
    a.act = static_cast<const uint16_t*>(act_bf16);
    a.lda = lda;
    a.act_gs = gsA_out;
    return from_cuda(fp4::launch_gemm_decode(a, dev, s));
}

fp4_status fp4_gemm_decode_noalloc(fp4_format fmt, const void* A, const void* sA, const void* B,
                                   const void* sB, int64_t M, int64_t N, int64_t K,
                                   const float* alpha, void* D, int64_t ldd, fp4_stream_t stream)
{
    fp4::g_last_error[0] = 0;
    if (!valid_fmt(fmt)) return FP4_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0) return FP4_ERR_INVALID_ARG;
    if (M > 16) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0 || K == 0)   // nothing that needs scratch
        return fp4_gemm_with_kernel(fmt, A, sA, B, sB, M, N, K, alpha, D, ldd, nullptr, 0,
                                    FP4_GEMM_PREFILL, stream);
    fp4::DeviceInfo dev;
    const fp4_status dst = require_device(&dev);
    if (dst != FP4_OK) return dst;
    const size_t need = fp4::decode_workspace_bytes(M, N, K, dev.sm_count);
    if (need == 0) {
        snprintf(fp4::g_last_error, sizeof fp4::g_last_error,
                 "N = %lld is beyond the decode kernel's arrival counters (N <= 524288)", (long long)N);
        return FP4_ERR_UNSUPPORTED_SHAPE;
    }
    if (need > fp4::noalloc_scratch_bytes()) {
        snprintf(fp4::g_last_error, sizeof fp4::g_last_error,
                 "decode partials need %zu bytes, above the %zu-byte static scratch", need,
                 fp4::noalloc_scratch_bytes());
        return FP4_ERR_UNSUPPORTED_SHAPE;
    }
    void* scratch = nullptr;
    const cudaError_t e = fp4::noalloc_scratch(&scratch);
    if (e != cudaSuccess) {
        fp4::set_last_error("cudaGetSymbolAddress(static decode scratch)", e);
        return from_cuda(e);
    }
    return fp4_gemm_with_kernel(fmt, A, sA, B, sB, M, N, K, alpha, D, ldd, scratch,
                                fp4::noalloc_scratch_bytes(), FP4_GEMM_DECODE, stream);
}

fp4_status fp4_selftest_bounded_wait(fp4_stream_t stream)
{
    fp4::g_last_error[0] = 0;
    fp4::DeviceInfo dev;
    fp4_status st = require_device(&dev);
    if (st != FP4_OK) return st;
    return from_cuda(fp4::launch_wait_selftest(reinterpret_cast<cudaStream_t>(stream)));
}

fp4_status fp4_get_device_status(fp4_stream_t stream)
{
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return from_cuda(e);
    unsigned int word = 0;
    e = fp4::read_and_clear_error_word(&word);
    if (e != cudaSuccess) return from_cuda(e);
    if (!word) return FP4_OK;
    e = fp4::clear_noalloc_counters(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return from_cuda(e);
    return (word & fp4::kErrorWorkspaceBit) && !(word & ~fp4::kErrorWorkspaceBit) ? FP4_ERR_WORKSPACE
                                                                                     : FP4_ERR_TIMEOUT;
}

}  // extern "C"
