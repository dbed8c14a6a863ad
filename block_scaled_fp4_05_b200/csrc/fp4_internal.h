// Host-side declarations shared by the translation units of libfp4.
#pragma once

#include <cstdint>
#include <cstddef>
#include <cuda_runtime.h>

#include "../../include/fp4.h"

namespace fp4 {

constexpr int kNv = 0;
constexpr int kMx = 1;
constexpr int kP1 = 2;   // 16-element blocks, E8M0 scale under S_global

inline int block_size(int fmt) { return fmt == kMx ? 32 : 16; }

// Device properties cached per device ordinal.
struct DeviceInfo {
    int sm_count = 0;
    int major = 0;
    int minor = 0;
};
cudaError_t device_info(DeviceInfo* out);

// quantize.cu
// S_global of x (and alpha = S_global * *other_gs when alpha_out is set) in
// one launch.
cudaError_t launch_global_scale(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                                float* gs_out, const float* other_gs, float* alpha_out,
                                cudaStream_t s);
// S_global of two tensors and alpha = gs_a * gs_b (alpha_out may be NULL) in
// one launch.
cudaError_t launch_global_scale_pair(const uint16_t* xa, int64_t rows_a, int64_t cols_a, int64_t ld_a,
                                     const uint16_t* xb, int64_t rows_b, int64_t cols_b, int64_t ld_b,
                                     float* gs_a, float* gs_b, float* alpha_out, cudaStream_t s);
cudaError_t launch_alpha(const float* gsA, const float* gsB, float* alpha, cudaStream_t s);
cudaError_t launch_quantize_dynamic(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                                    uint8_t* packed, uint8_t* scales, float* gs_out,
                                    const float* other_gs, float* alpha_out, cudaStream_t s);
cudaError_t launch_quantize(int fmt, int axis, const uint16_t* x, int64_t rows, int64_t cols,
                            int64_t ld, uint8_t* packed, uint8_t* scales, const float* gs,
                            cudaStream_t s);
cudaError_t launch_dequantize(int fmt, const uint8_t* packed, const uint8_t* scales, const float* gs,
                              int64_t rows, int64_t k, uint16_t* out, int64_t ld, cudaStream_t s);
// Rowwise quantization of n tensors, batched into one launch per 8.
struct RowwiseDesc {
    const uint16_t* x;
    int64_t rows, cols, ld;
    uint8_t* packed;
    uint8_t* scales;
    const float* gs;   // NVFP4 S_global, NULL for MXFP4
};
// reverse: the tiles run last to first (same results).
cudaError_t launch_quantize_rowwise_batch(int fmt, int n, const RowwiseDesc* d, cudaStream_t s,
                                          bool reverse = false);

// gemm.cu
struct GemmArgs {
    int fmt;
    const uint8_t* A;   // [M x K/2]
    const uint8_t* sA;
    const uint8_t* B;   // [N x K/2]
    const uint8_t* sB;
    int64_t M, N, K;
    const float* alpha;
    uint16_t* D;        // bf16 [M x N], ldd
    int64_t ldd;
    void* ws;
    size_t ws_bytes;
    bool b_static;      // B and sB not written by a kernel still running on the stream
    // decode form only: the activation as BF16 [M x K] (leading dimension
    // lda), quantized inside the GEMM with S_global *act_gs (A and sA unused)
    const uint16_t* act = nullptr;
    int64_t lda = 0;
    const float* act_gs = nullptr;
};
size_t decode_workspace_bytes(int64_t M, int64_t N, int64_t K, int sm_count);
cudaError_t launch_gemm_prefill(const GemmArgs& a, const DeviceInfo& dev, cudaStream_t s);
cudaError_t launch_gemm_decode(const GemmArgs& a, const DeviceInfo& dev, cudaStream_t s);
cudaError_t launch_gemm_grouped(int n, const GemmArgs* a, const DeviceInfo& dev, cudaStream_t s);
cudaError_t read_and_clear_error_word(unsigned int* word);
cudaError_t launch_wait_selftest(cudaStream_t s);
size_t noalloc_scratch_bytes();
cudaError_t noalloc_scratch(void** out);
// Zeroes the decode counters of the static scratch (current device), after an
// error left them in an unknown state: a memset on stream s, then a wait for s.
cudaError_t clear_noalloc_counters(cudaStream_t s);
// The calling thread's current CUDA context (driver handle, as an opaque
// pointer), for caches of per-context device addresses.
cudaError_t current_context(void** ctx);
// Bit of the device error word set by a decode call whose workspace counters
// were out of range (not zeroed).
constexpr unsigned int kErrorWorkspaceBit = 64u;
int tensor_map_encoder_available();

// Records the detail of a failure for fp4_last_error() (thread-local).
void set_last_error(const char* what, cudaError_t e);
extern thread_local char g_last_error[256];

}  // namespace fp4
