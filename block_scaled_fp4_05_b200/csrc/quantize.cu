// Block quantizer kernels: BF16 -> E2M1 codes + per-block scales (NVFP4,
// MXFP4, and 16-element blocks with E8M0 scales under S_global) for one
// tensor or a batch (one launch over the tiles of up to 8 tensors), the
// per-tensor amax for S_global, alpha = gsA * gsB, the one-launch dynamic
// quantization of a small activation, and the reconstruction to BF16.
//
// Method: "NVFP4 Architecture: Microscaling & 4-Bit LLMs on Blackwell",
// "1. The Dual-Level Mathematical Formulation" (S_global, S_block,j, q_i) and
// the emulation script of "End-to-End Implementation" (block amax, 1e-8
// clamp, S = 2^ceil(log2(amax/6)), nearest E2M1 value); MXFP4 block size and
// E8M0 scale from "MXFP4" / "Core Facts".
//
// The kernels are HBM-bound (2 B read, 0.5 + 1/k B written per element).
// One CTA owns one 128-row x 4-block tile of the output, which is exactly one
// 512-byte scale tile in the MMA layout, so the scale bytes are assembled in
// shared memory and written as one coalesced 512-byte chunk.  Inputs are read
// with 128-bit streaming loads, 8 BF16 per thread per load; the block amax is
// an integer max over BF16 magnitude bits, combined across the 2 (k=16) or 4
// (k=32) lanes of a block with warp shuffles.

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <cfloat>
#include <mutex>

#include "fp4_internal.h"
#include "quant_device.cuh"

namespace fp4 {
namespace {

using namespace qdev;

constexpr int kThreads = 256;
constexpr int kMaxBatch = 8;   // tensors per batched launch

// Lets a kernel launched after this one with programmatic stream
// serialization (the GEMMs) start its set-up; it still waits for this
// kernel's completion before reading anything this kernel writes.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Rowwise: CTA tile = 128 rows x 4k columns -> one 512-byte scale tile.
// grid = (cols / 4k, ceil(rows / 128)).
// ---------------------------------------------------------------------------
template <int FMT>
__device__ __forceinline__ void rowwise_tile(const uint16_t* __restrict__ x, int64_t rows, int64_t cols,
                                             int64_t ld, uint8_t* __restrict__ packed,
                                             uint8_t* __restrict__ scales, int64_t rt, int64_t ct,
                                             float gs, float denom, uint8_t* s_tile)
{
    constexpr int KB = FMT == kMx ? 32 : 16;     // elements per block
    constexpr int TILE_C = 4 * KB;               // columns per tile
    constexpr int CPR = TILE_C / 8;              // 16-byte chunks per row
    constexpr int RPP = kThreads / CPR;          // rows per pass
    constexpr int PASSES = 128 / RPP;
    constexpr int CPB = KB / 8;                  // chunks per block

    const int tid = threadIdx.x;
    const int cc = tid % CPR;
    const int rsub = tid / CPR;
    const int64_t c0 = ct * TILE_C;
    const int64_t r0 = rt * 128;
    const int64_t nct = cols / TILE_C;

    uint4 v[PASSES];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int64_t r = r0 + rsub + p * RPP;
        if (r < rows)
            v[p] = ld_stream(reinterpret_cast<const uint4*>(x + r * ld + c0) + cc);
        else
            v[p] = make_uint4(0u, 0u, 0u, 0u);
    }

    uint32_t* out32 = reinterpret_cast<uint32_t*>(packed);
    const int64_t row_words = cols / 8;  // 4-byte words per packed row
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int rl = rsub + p * RPP;
        const int64_t r = r0 + rl;
        uint32_t am = absmax8(v[p]);
        if (CPB >= 2) am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
        if (CPB >= 4) am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 2));
        float inv;
        const uint32_t sbyte = block_scale<FMT>(am, gs, denom, &inv);
        const uint32_t q = quantize8(v[p], inv);
        if (r < rows)
            out32[r * row_words + c0 / 8 + cc] = q;
        if (cc % CPB == 0)
            s_tile[(rl % 32) * 16 + (rl / 32) * 4 + cc / CPB] = (r < rows) ? (uint8_t)sbyte : 0;
    }
    __syncthreads();
    if (tid < 32) {
        const uint4 t = reinterpret_cast<const uint4*>(s_tile)[tid];
        reinterpret_cast<uint4*>(scales + (rt * nct + ct) * 512)[tid] = t;
    }
}

// The tile list of a batch of tensors: tile t belongs to tensor k with
// tile_begin[k] <= t < tile_begin[k+1]; within a tensor, column tiles run
// fastest.  Used by both rowwise kernels (with their own tile widths).
struct RowBatch {
    int n;
    int reverse;                         // tiles in reverse order (last tile first)
    int64_t tile_begin[kMaxBatch + 1];   // prefix sums of the tensors' tile counts
    const uint16_t* x[kMaxBatch];
    int64_t rows[kMaxBatch], cols[kMaxBatch], ld[kMaxBatch];
    uint8_t* packed[kMaxBatch];
    uint8_t* scales[kMaxBatch];
    const float* gs[kMaxBatch];
};

__device__ __forceinline__ void locate_tile(const RowBatch& b, int64_t t, int64_t tile_c, int& k,
                                            int64_t& rt, int64_t& ct)
{
    k = 0;
    while (t >= b.tile_begin[k + 1]) ++k;
    const int64_t local = t - b.tile_begin[k];
    const int64_t nct = (b.cols[k] + tile_c - 1) / tile_c;
    rt = local / nct;
    ct = local - rt * nct;
}

// One CTA per 128-row x 4-block tile: grid = all tiles of the batch.
template <int FMT>
__global__ void __launch_bounds__(kThreads)
quantize_rowwise_tiles_kernel(const __grid_constant__ RowBatch b)
{
    __shared__ __align__(16) uint8_t s_tile[512];
    pdl_trigger();
    constexpr int TILE_C = 4 * (FMT == kMx ? 32 : 16);
    int k;
    int64_t rt, ct;
    locate_tile(b, b.reverse ? gridDim.x - 1 - blockIdx.x : blockIdx.x, TILE_C, k, rt, ct);
    float gs = 1.0f, denom = 6.0f;
    if (FMT != kMx) {
        gs = __ldg(b.gs[k]);
        denom = __fmul_rn(6.0f, gs);
    }
    rowwise_tile<FMT>(b.x[k], b.rows[k], b.cols[k], b.ld[k], b.packed[k], b.scales[k], rt, ct, gs, denom,
                      s_tile);
}

// ---------------------------------------------------------------------------
// Dequantization (reconstruction) x_hat = q * S_block (* S_global) of a
// rowwise-quantized operand [rows x k] into BF16, rounded once to nearest
// even: the product of the E2M1 value, the block scale and S_global is exact
// in FP64 (at most 2 + 4 + 24 significant bits), then converted.  HBM-bound
// (0.5 + 1/blk bytes read, 2 written per element).
// Each block first tabulates, for all 256 scale bytes, the BF16 results of
// the eight E2M1 magnitudes times that scale (exact FP64 product, one
// rounding): the low bytes of magnitudes 0..7 in 8 bytes, the high bytes in
// 8 more.  A code's magnitude (3 bits) is then directly a byte-permute
// selector: one permute yields the high (or low) bytes of four codes, the
// code signs flip bit 7 of the high bytes, and two more permutes interleave
// low and high bytes into BF16 pairs.
// A warp takes 2048 consecutive codes of one row (8 segments of 256): in each
// segment lane l owns codes [8l, 8l + 8), one 4-byte load of packed codes and
// one 16-byte store of BF16, so every warp load covers 128 contiguous bytes
// and every warp store 512.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t bf16_bits_rn(double x)
{
    unsigned short h;
    asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(h) : "d"(x));
    return h;
}

// Eight E2M1 codes (code i in bits 4i..4i+3 of w) to BF16 through the table
// entry tb of their block's scale byte (x, y: low bytes of magnitudes 0..3,
// 4..7; z, w: high bytes): output word i holds codes 2i (low half) and 2i + 1.
__device__ __forceinline__ uint4 decode8(uint32_t w, uint4 tb)
{
    const uint32_t sel0 = w & 0x7777u;            // magnitudes of codes 0..3
    const uint32_t sel1 = (w >> 16) & 0x7777u;    // codes 4..7
    const uint32_t l0 = __byte_perm(tb.x, tb.y, sel0), l1 = __byte_perm(tb.x, tb.y, sel1);
    uint32_t h0 = __byte_perm(tb.z, tb.w, sel0), h1 = __byte_perm(tb.z, tb.w, sel1);
    // sign of code 2j (2j + 1) in bit 7 of byte j of ev (od)
    const uint32_t ev = (w << 4) & 0x80808080u, od = w & 0x80808080u;
    h0 ^= __byte_perm(ev, od, 0x5140);
    h1 ^= __byte_perm(ev, od, 0x7362);
    return make_uint4(__byte_perm(l0, h0, 0x5140), __byte_perm(l0, h0, 0x7362), __byte_perm(l1, h1, 0x5140),
                      __byte_perm(l1, h1, 0x7362));
}

template <int FMT>
__global__ void __launch_bounds__(kThreads)
dequantize_kernel(const uint8_t* __restrict__ packed, const uint8_t* __restrict__ scales,
                  const float* __restrict__ gs_ptr, int64_t rows, int64_t k, uint16_t* __restrict__ out,
                  int64_t ld)
{
    static_assert(kThreads == 256, "one table entry per thread");
    pdl_trigger();
    constexpr int KB = FMT == kMx ? 32 : 16;
    constexpr int CPT = 4 * KB;                         // codes per 512-byte scale tile column
    constexpr int SEG = 256;                            // codes per warp segment
    constexpr int UNROLL = 8;
    __shared__ uint4 s_tab[256];
    {
        const uint32_t byte = threadIdx.x;
        const double gs = FMT != kMx ? (double)__ldg(gs_ptr) : 1.0;
        const double s = FMT == kNv ? (double)e4m3_value(byte)
                                    : __longlong_as_double((long long)(byte + 896) << 52);  // 2^(byte - 127)
        const double eff = s * gs;
        const double q[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
        uint32_t lo[2] = {0u, 0u}, hi[2] = {0u, 0u};
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const uint32_t b = bf16_bits_rn(q[m] * eff);
            lo[m / 4] |= (b & 0xFFu) << (8 * (m % 4));
            hi[m / 4] |= (b >> 8) << (8 * (m % 4));
        }
        s_tab[byte] = make_uint4(lo[0], lo[1], hi[0], hi[1]);
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t nct = (k / KB + 3) / 4;               // scale tile columns per 128-row group
    const int64_t groups_per_row = (k + SEG * UNROLL - 1) / (SEG * UNROLL);
    const int64_t total = rows * groups_per_row;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    // this lane's scale byte within a segment: tile column, then block in it
    const int lane_sc = ((lane * 8) / CPT) * 512 + ((lane * 8) / KB) % 4;
    for (int64_t w = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); w < total; w += warps) {
        const int64_t r = w / groups_per_row;
        const int c_base = (int)(w - r * groups_per_row) * (SEG * UNROLL);
        const uint32_t* prow = reinterpret_cast<const uint32_t*>(packed + r * (k / 2) + c_base / 2) + lane;
        const uint8_t* srow = scales + (r / 128) * nct * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 +
                              (int64_t)(c_base / CPT) * 512 + lane_sc;
        uint16_t* orow = out + r * ld + c_base + lane * 8;
        const int64_t rem = k - c_base;                 // codes of the row from c_base on
        const int left = (int)(rem < SEG * UNROLL ? rem : SEG * UNROLL) - lane * 8;
        uint32_t words[UNROLL];
        uint32_t sbytes[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const bool in = u * SEG < left;
            words[u] = in ? __ldg(prow + u * (SEG / 8)) : 0u;
            sbytes[u] = in ? __ldg(srow + u * (SEG / CPT) * 512) : 0u;
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u)
            if (u * SEG < left) *reinterpret_cast<uint4*>(orow + u * SEG) = decode8(words[u], s_tab[sbytes[u]]);
    }
}

// ---------------------------------------------------------------------------
// Dynamic NVFP4 quantization of a small tensor (decode activations) in one
// launch: a cluster of CTAs reads the tensor once into registers, computes
// its amax (each CTA's partial maximum stored into every CTA's shared memory
// through DSMEM, one cluster barrier), S_global =
// amax / 2688 (1 for an all-zero tensor) and optionally alpha = S_global *
// other, then quantizes the register-resident values with that scale.
// Thread t of the cluster owns the 16-byte chunks t, t + T, t + 2T, ... of the
// row-major tensor (T = threads in the cluster), so every warp load and store
// is contiguous; a lane pair holds one 16-element block and eight lanes one
// 4-byte group of a scale tile.  Padding rows of the last 128-row scale tile
// get zero scale bytes, written while the loads are in flight.  Tensors with
// more chunks than the cluster holds in registers take the amax / quantize /
// alpha kernels instead (launch_quantize_dynamic).
// ---------------------------------------------------------------------------
constexpr int kDynClusterMax = 16;   // non-portable size, used when the device can schedule it
constexpr int kDynClusterMin = 8;
constexpr int kDynThreads = 512;    // leaves room on the SM for a GEMM CTA launched early
constexpr int kDynRegChunks = 4;

__global__ void __launch_bounds__(kDynThreads)
quantize_dynamic_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                        uint8_t* __restrict__ packed, uint8_t* __restrict__ scales,
                        float* __restrict__ gs_out, const float* __restrict__ other_gs,
                        float* __restrict__ alpha_out)
{
    __shared__ uint32_t s_part[kDynClusterMax];
    __shared__ uint32_t s_warp[kDynThreads / 32];
    __shared__ float s_gs;

    pdl_trigger();
    uint32_t rank, csize;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(csize));
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    // chunk indices fit 32 bits (at most kDynMaxChunks chunks)
    const uint32_t T = csize * kDynThreads;
    const uint32_t gt = rank * kDynThreads + tid;
    const uint32_t cpr = (uint32_t)(cols / 8);     // 16-byte chunks per row = packed words per row
    const uint32_t n = (uint32_t)rows * cpr;
    const uint32_t G = cpr / 8;                    // scale groups per row
    auto scale_word = [&](uint32_t r, uint32_t g) {
        return reinterpret_cast<uint32_t*>(scales + ((size_t)(r / 128) * G + g) * 512 + (r % 32) * 16 +
                                           ((r / 32) % 4) * 4);
    };

    // phase 1: load this thread's chunks, amax over the cluster
    uint4 v[kDynRegChunks];
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < kDynRegChunks; ++j) {
        const uint32_t u = j * T + gt;
        v[j] = make_uint4(0u, 0u, 0u, 0u);
        if (u < n) {
            const uint32_t r = u / cpr;
            v[j] = ld_stream(reinterpret_cast<const uint4*>(x + (int64_t)r * ld) + (u - r * cpr));
        }
    }
    // zero scale bytes for the padding rows of the last 128-row tile:
    // consecutive threads take consecutive words of a 512-byte scale tile
    // (word k holds row (k % 4) * 32 + k / 4 of the tile)
    {
        const uint32_t rt = (uint32_t)(rows - 1) / 128, first_pad = (uint32_t)rows - rt * 128;
        if (first_pad < 128) {
            uint32_t* tile0 = reinterpret_cast<uint32_t*>(scales + (size_t)rt * G * 512);
            for (uint32_t w = gt; w < G * 128; w += T) {
                const uint32_t k = w % 128;
                if ((k % 4) * 32 + k / 4 >= first_pad) tile0[w] = 0u;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kDynRegChunks; ++j) m = max(m, absmax8(v[j]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) s_warp[tid >> 5] = m;
    __syncthreads();
    // every CTA's partial max goes to every CTA, so that after the barrier
    // the maxima are read locally and no CTA touches another's shared
    // memory again
    if (tid < (int)csize) {
        uint32_t b = 0;
        for (int w = 0; w < kDynThreads / 32; ++w) b = max(b, s_warp[w]);
        uint32_t dst;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(dst)
                     : "r"((uint32_t)__cvta_generic_to_shared(&s_part[rank])), "r"(tid));
        asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(dst), "r"(b) : "memory");
    }
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
    if (tid == 0) {
        uint32_t b = 0;
        for (uint32_t i = 0; i < csize; ++i) b = max(b, s_part[i]);
        const float amax = __uint_as_float(b << 16);
        const float gs = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
        s_gs = gs;
        if (rank == 0) {
            *gs_out = gs;
            if (alpha_out) *alpha_out = __fmul_rn(gs, __ldg(other_gs));
        }
    }
    __syncthreads();
    const float gs = s_gs;
    const float denom = __fmul_rn(6.0f, gs);

    // phase 2: quantize the register-resident chunks
    uint32_t* out32 = reinterpret_cast<uint32_t*>(packed);
    const int gbase = lane & ~7;
#pragma unroll
    for (int j = 0; j < kDynRegChunks; ++j) {
        const uint32_t u = j * T + gt;
        if (j * T + (gt & ~31u) >= n) break;   // warp-uniform: no chunk of this warp left
        uint32_t am = absmax8(v[j]);
        am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
        float inv;
        const uint32_t sb = block_scale<kNv>(am, gs, denom, &inv);
        const uint32_t q = quantize8(v[j], inv);
        const uint32_t word = __shfl_sync(0xFFFFFFFFu, sb, gbase) |
                              (__shfl_sync(0xFFFFFFFFu, sb, gbase + 2) << 8) |
                              (__shfl_sync(0xFFFFFFFFu, sb, gbase + 4) << 16) |
                              (__shfl_sync(0xFFFFFFFFu, sb, gbase + 6) << 24);
        if (u < n) {
            out32[u] = q;
            if ((lane & 7) == 0) {
                const uint32_t r = u / cpr;
                *scale_word(r, (u - r * cpr) / 8) = word;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Colwise: blocks run down the columns; output row c = input column c.
// CTA tile = 4k input rows (the blocked direction) x 128 input columns (the
// output rows) -> one 512-byte scale tile.  The BF16 tile is staged through
// shared memory, each thread then quantizes whole blocks (one column, k
// consecutive rows), and the packed output tile is staged again so that the
// global writes are coalesced.  grid = (rows / 4k, ceil(cols / 128)).
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void __launch_bounds__(kThreads)
quantize_colwise_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                        uint8_t* __restrict__ packed, uint8_t* __restrict__ scales,
                        const float* __restrict__ gs_ptr)
{
    constexpr int KB = FMT == kMx ? 32 : 16;
    constexpr int TILE_K = 4 * KB;                       // input rows per CTA
    constexpr int LOAD_PASSES = TILE_K * 16 / kThreads;  // 16 chunks of 8 per input row
    constexpr int OUT_BYTES = TILE_K / 2;                // packed bytes per output row

    __shared__ __align__(16) uint16_t s_in[TILE_K][128];
    __shared__ __align__(16) uint8_t s_out[128][OUT_BYTES];
    __shared__ __align__(16) uint8_t s_tile[512];
    pdl_trigger();

    const int tid = threadIdx.x;
    const int64_t kt = blockIdx.x;        // scale-column tile (blocked direction)
    const int64_t ot = blockIdx.y;        // output row tile
    const int64_t k0 = kt * TILE_K;
    const int64_t oc0 = ot * 128;
    const int64_t nct = rows / TILE_K;

    float gs = 1.0f, denom = 6.0f;
    if (FMT != kMx) {
        gs = __ldg(gs_ptr);
        denom = __fmul_rn(6.0f, gs);
    }

    // coalesced load of the TILE_K x 128 BF16 tile (zero past the last column)
#pragma unroll
    for (int p = 0; p < LOAD_PASSES; ++p) {
        const int lr = tid / 16 + p * (kThreads / 16);
        const int ch = tid % 16;
        const int64_t c = oc0 + ch * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (c < cols)
            v = ld_stream(reinterpret_cast<const uint4*>(x + (k0 + lr) * ld + c));
        *reinterpret_cast<uint4*>(&s_in[lr][ch * 8]) = v;
    }
    __syncthreads();

    // each thread: 2 blocks (output row o, block b); a warp covers 32
    // consecutive output rows of one block, so shared reads are conflict-free
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int task = tid + i * kThreads;
        const int o = task % 128;
        const int b = task / 128;
        uint32_t w[KB / 2];
        uint32_t am = 0;
#pragma unroll
        for (int j = 0; j < KB / 2; ++j) {
            const uint32_t lo = s_in[b * KB + 2 * j][o];
            const uint32_t hi = s_in[b * KB + 2 * j + 1][o];
            w[j] = lo | (hi << 16);
            am = max(am, max(lo & 0x7FFFu, hi & 0x7FFFu));
        }
        float inv;
        const uint32_t sbyte = block_scale<FMT>(am, gs, denom, &inv);
#pragma unroll
        for (int j = 0; j < KB / 8; ++j) {
            const uint4 v = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
            *reinterpret_cast<uint32_t*>(&s_out[o][b * (KB / 2) + 4 * j]) = quantize8(v, inv);
        }
        const bool valid = (oc0 + o) < cols;
        s_tile[(o % 32) * 16 + (o / 32) * 4 + b] = valid ? (uint8_t)sbyte : 0;
    }
    __syncthreads();

    // packed rows: OUT_BYTES per output row, 16 bytes per thread
    constexpr int CH_PER_ROW = OUT_BYTES / 16;
    const int64_t out_row_bytes = rows / 2;
#pragma unroll
    for (int p = 0; p < (128 * CH_PER_ROW) / kThreads; ++p) {
        const int idx = tid + p * kThreads;
        const int o = idx / CH_PER_ROW;
        const int ch = idx % CH_PER_ROW;
        if (oc0 + o < cols) {
            const uint4 t = *reinterpret_cast<const uint4*>(&s_out[o][ch * 16]);
            *reinterpret_cast<uint4*>(packed + (oc0 + o) * out_row_bytes + k0 / 2 + ch * 16) = t;
        }
    }
    if (tid < 32) {
        const uint4 t = reinterpret_cast<const uint4*>(s_tile)[tid];
        reinterpret_cast<uint4*>(scales + (ot * nct + kt) * 512)[tid] = t;
    }
}

// ---------------------------------------------------------------------------
// S_global = amax / 2688 (1 when amax == 0) of a BF16 matrix, and optionally
// alpha = S_global * other, in one launch.  Each CTA reduces its share of the
// rows to one BF16 magnitude (an integer max over the magnitude bits) and
// folds it into a reduction slot with atomicMax; the CTA whose arrival on the
// slot's counter is the last one finalizes: it reads the slot's maximum,
// writes S_global (and alpha) and resets the slot to zero for its next use.
// The slots live in a ring in static device memory, zero at load; each call
// takes the next slot, so calls in flight at the same time (other streams)
// reduce into different slots.
// ---------------------------------------------------------------------------
struct GsSlot {
    unsigned int amax[2];   // BF16 magnitude bits of each tensor
    unsigned int count;     // CTAs arrived
    unsigned int pad;
};
constexpr int kGsSlots = 1024;
__device__ GsSlot g_gs_slots[kGsSlots];

constexpr int kGsUnroll = 8;   // 16-byte loads in flight per thread

// One or two tensors per launch.  Each tensor's rows are split into segments
// of kThreads * kGsUnroll chunks (8 BF16 each), segment s of the launch
// belonging to tensor 1 from seg_begin1 on; the CTAs take segments in a
// grid-stride loop, so no per-load index division is needed.  A contiguous
// matrix (ld == cols) is one long row.
struct GsArgs {
    const uint16_t* x[2];
    int64_t cpr[2], ld[2], spr[2];
    int64_t seg_begin1, seg_total;
    float* gs_out[2];
    const float* other_gs;   // one tensor: alpha = gs * *other_gs (if alpha_out)
    float* alpha_out;        // two tensors: alpha = gs[0] * gs[1] (if alpha_out)
    int n;
};

__global__ void __launch_bounds__(kThreads)
global_scale_kernel(const __grid_constant__ GsArgs a, GsSlot* __restrict__ slot)
{
    pdl_trigger();
    uint32_t m0 = 0u, m1 = 0u;   // the two tensors' maxima (registers, not an indexed array)
    for (int64_t sidx = blockIdx.x; sidx < a.seg_total; sidx += gridDim.x) {
        const int k = sidx >= a.seg_begin1 ? 1 : 0;
        const int64_t ls = sidx - (k ? a.seg_begin1 : 0);
        const int64_t r = ls / a.spr[k];
        const int64_t c0 = (ls - r * a.spr[k]) * (kThreads * kGsUnroll) + threadIdx.x;
        const uint4* row = reinterpret_cast<const uint4*>(a.x[k] + r * a.ld[k]);
        uint4 v[kGsUnroll];
#pragma unroll
        for (int u = 0; u < kGsUnroll; ++u) {
            const int64_t c = c0 + u * kThreads;
            v[u] = c < a.cpr[k] ? ld_stream(row + c) : make_uint4(0u, 0u, 0u, 0u);
        }
        uint32_t mm = 0;
#pragma unroll
        for (int u = 0; u < kGsUnroll; ++u) mm = max(mm, absmax8(v[u]));
        if (k) m1 = max(m1, mm); else m0 = max(m0, mm);
    }
    uint32_t m[2] = {m0, m1};
    __shared__ uint32_t s_m[2][kThreads / 32];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m[k] = max(m[k], __shfl_xor_sync(0xFFFFFFFFu, m[k], o));
        if ((threadIdx.x & 31) == 0) s_m[k][threadIdx.x >> 5] = m[k];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int k = 0; k < a.n; ++k) {
            uint32_t b = 0;
            for (int w = 0; w < kThreads / 32; ++w) b = max(b, s_m[k][w]);
            if (b) atomicMax(&slot->amax[k], b);
        }
        // release: this CTA's maxima are visible before its arrival counts;
        // acquire: the last arriver sees every other CTA's maxima
        unsigned int old;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                     : "=r"(old) : "l"(&slot->count) : "memory");
        if (old == gridDim.x - 1) {
            float gs[2] = {1.0f, 1.0f};
            for (int k = 0; k < a.n; ++k) {
                unsigned int bits;
                asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(bits) : "l"(&slot->amax[k]) : "memory");
                const float amax = __uint_as_float(bits << 16);
                gs[k] = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
                *a.gs_out[k] = gs[k];
                slot->amax[k] = 0u;
            }
            if (a.alpha_out) *a.alpha_out = __fmul_rn(gs[0], a.n == 2 ? gs[1] : *a.other_gs);
            slot->count = 0u;
        }
    }
}

__global__ void alpha_kernel(const float* a, const float* b, float* out)
{
    *out = __fmul_rn(*a, *b);
}

// Device address of the slot ring in the current context (looked up once per
// device and context: in host code the array's name is not a device address).
cudaError_t gs_slots(GsSlot** out)
{
    static std::mutex mu;
    static GsSlot* cache[64] = {};
    static void* cache_ctx[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    void* ctx = nullptr;
    e = current_context(&ctx);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && cache[dev] && cache_ctx[dev] == ctx) {
        *out = cache[dev];
        return cudaSuccess;
    }
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(out), g_gs_slots);
    if (e == cudaSuccess && dev < 64) {
        cache[dev] = *out;
        cache_ctx[dev] = ctx;
    }
    return e;
}

}  // namespace

cudaError_t launch_alpha(const float* gsA, const float* gsB, float* alpha, cudaStream_t s)
{
    alpha_kernel<<<1, 1, 0, s>>>(gsA, gsB, alpha);
    return cudaGetLastError();
}

// Segments of one tensor: a contiguous matrix (ld == cols) is reduced as one
// row.
static void gs_tensor(GsArgs& a, int k, const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                      float* gs_out, int64_t* nseg)
{
    const bool flat = ld == cols;
    const int64_t r = flat ? 1 : rows;
    a.x[k] = x;
    a.cpr[k] = flat ? rows * cols / 8 : cols / 8;
    a.ld[k] = ld;
    a.spr[k] = (a.cpr[k] + kThreads * kGsUnroll - 1) / (kThreads * kGsUnroll);
    a.gs_out[k] = gs_out;
    *nseg = (rows == 0 || cols == 0) ? 0 : r * a.spr[k];
}

// Resident CTAs per SM of the S_global kernel (per device, looked up once).
static int global_scale_blocks_per_sm()
{
    static std::mutex mu;
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 4;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && cache[dev]) return cache[dev];
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, global_scale_kernel, kThreads, 0) != cudaSuccess ||
        nb < 1) {
        cudaGetLastError();
        nb = 4;
    }
    if (dev < 64) cache[dev] = nb;
    return nb;
}

static cudaError_t launch_gs(GsArgs& a, int64_t seg0, int64_t seg1, cudaStream_t s)
{
    static unsigned int next_slot = 0;   // ring position (atomic: calls from several threads)
    DeviceInfo dev;
    cudaError_t e = device_info(&dev);
    if (e != cudaSuccess) return e;
    GsSlot* slots = nullptr;
    e = gs_slots(&slots);
    if (e != cudaSuccess) return e;
    const unsigned int k = __atomic_fetch_add(&next_slot, 1u, __ATOMIC_RELAXED) % kGsSlots;
    a.seg_begin1 = seg0;
    a.seg_total = seg0 + seg1;
    int64_t grid = a.seg_total;
    // one wave: every CTA resident from the start, segments taken grid-stride
    const int64_t cap = (int64_t)dev.sm_count * global_scale_blocks_per_sm();
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    global_scale_kernel<<<(unsigned)grid, kThreads, 0, s>>>(a, slots + k);
    return cudaGetLastError();
}

cudaError_t launch_global_scale(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                                float* gs_out, const float* other_gs, float* alpha_out,
                                cudaStream_t s)
{
    GsArgs a = {};
    int64_t n0 = 0;
    gs_tensor(a, 0, x, rows, cols, ld, gs_out, &n0);
    a.n = 1;
    a.other_gs = other_gs;
    a.alpha_out = alpha_out;
    return launch_gs(a, n0, 0, s);
}

cudaError_t launch_global_scale_pair(const uint16_t* xa, int64_t rows_a, int64_t cols_a, int64_t ld_a,
                                     const uint16_t* xb, int64_t rows_b, int64_t cols_b, int64_t ld_b,
                                     float* gs_a, float* gs_b, float* alpha_out, cudaStream_t s)
{
    GsArgs a = {};
    int64_t n0 = 0, n1 = 0;
    gs_tensor(a, 0, xa, rows_a, cols_a, ld_a, gs_a, &n0);
    gs_tensor(a, 1, xb, rows_b, cols_b, ld_b, gs_b, &n1);
    a.n = 2;
    a.alpha_out = alpha_out;
    return launch_gs(a, n0, n1, s);
}

namespace {

// Cluster size for the dynamic quantizer: 16 CTAs when the device can place
// such a cluster, else the portable 8.  Decided once per device (the
// non-portable-size attribute is set on each device that uses it).
int dynamic_cluster_size()
{
    static std::mutex mu;
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return kDynClusterMin;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && cache[dev]) return cache[dev];
    int chosen = kDynClusterMin;
    if (cudaFuncSetAttribute(quantize_dynamic_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
        cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kDynClusterMax, 1, 1);
        cfg.blockDim = dim3(kDynThreads, 1, 1);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kDynClusterMax;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, quantize_dynamic_kernel, &cfg) == cudaSuccess && n >= 1)
            chosen = kDynClusterMax;
    }
    cudaGetLastError();
    if (dev < 64) cache[dev] = chosen;
    return chosen;
}

}  // namespace

cudaError_t launch_quantize_dynamic(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                                    uint8_t* packed, uint8_t* scales, float* gs_out,
                                    const float* other_gs, float* alpha_out, cudaStream_t s)
{
    const int cl = dynamic_cluster_size();
    if (rows * (cols / 8) > (int64_t)cl * kDynThreads * kDynRegChunks) {
        // too large to stay in one cluster's registers: S_global and alpha in
        // one launch, then the rowwise quantizer.  The quantizer takes its
        // tiles in reverse order: the amax pass ends at the tensor's last rows,
        // so those are still in L2 when the quantizer starts on them.
        cudaError_t e = launch_global_scale(x, rows, cols, ld, gs_out, other_gs, alpha_out, s);
        const RowwiseDesc d = {x, rows, cols, ld, packed, scales, gs_out};
        if (e == cudaSuccess) e = launch_quantize_rowwise_batch(kNv, 1, &d, s, true);
        if (e != cudaSuccess) set_last_error("dynamic quantizer (multi-kernel) launch", e);
        return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cl, 1, 1);
    cfg.blockDim = dim3(kDynThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, quantize_dynamic_kernel, x, rows, cols, ld, packed, scales,
                                       gs_out, other_gs, alpha_out);
    if (e != cudaSuccess) set_last_error("dynamic quantizer launch", e);
    return e;
}

// One launch over the tiles of up to kMaxBatch tensors.  (A persistent
// variant that streamed the tiles through a cp.async ring in shared memory
// was measured slower for both formats: one CTA per tile, many of them
// resident, keeps more loads in flight.)
cudaError_t launch_quantize_rowwise_batch(int fmt, int n, const RowwiseDesc* d, cudaStream_t s,
                                          bool reverse)
{
    const int64_t tile_c = 4 * block_size(fmt);
    for (int i0 = 0; i0 < n; i0 += kMaxBatch) {
        RowBatch b = {};
        b.n = 0;
        b.reverse = reverse ? 1 : 0;
        b.tile_begin[0] = 0;
        for (int i = i0; i < n && i < i0 + kMaxBatch; ++i) {
            if (d[i].rows == 0 || d[i].cols == 0) continue;
            const int j = b.n++;
            b.x[j] = d[i].x;
            b.rows[j] = d[i].rows;
            b.cols[j] = d[i].cols;
            b.ld[j] = d[i].ld;
            b.packed[j] = d[i].packed;
            b.scales[j] = d[i].scales;
            b.gs[j] = d[i].gs;
            b.tile_begin[j + 1] = b.tile_begin[j] + ((d[i].rows + 127) / 128) * ((d[i].cols + tile_c - 1) / tile_c);
        }
        if (b.n == 0) continue;
        const int64_t tiles = b.tile_begin[b.n];
        if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
        if (fmt == kNv)
            quantize_rowwise_tiles_kernel<kNv><<<(unsigned)tiles, kThreads, 0, s>>>(b);
        else if (fmt == kP1)
            quantize_rowwise_tiles_kernel<kP1><<<(unsigned)tiles, kThreads, 0, s>>>(b);
        else
            quantize_rowwise_tiles_kernel<kMx><<<(unsigned)tiles, kThreads, 0, s>>>(b);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// Resident blocks per SM of the dequantizer (per device and format, looked
// up once).
int dequantize_blocks_per_sm(int fmt)
{
    static std::mutex mu;
    static int cache[64][3] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 4;
    }
    const int f = fmt == kNv ? 0 : fmt == kP1 ? 1 : 2;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && cache[dev][f]) return cache[dev][f];
    int nb = 0;
    cudaError_t e = fmt == kNv ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, dequantize_kernel<kNv>, kThreads, 0)
                  : fmt == kP1 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, dequantize_kernel<kP1>, kThreads, 0)
                               : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, dequantize_kernel<kMx>, kThreads, 0);
    if (e != cudaSuccess || nb < 1) {
        cudaGetLastError();
        nb = 4;
    }
    if (dev < 64) cache[dev][f] = nb;
    return nb;
}

cudaError_t launch_dequantize(int fmt, const uint8_t* packed, const uint8_t* scales, const float* gs,
                              int64_t rows, int64_t k, uint16_t* out, int64_t ld, cudaStream_t s)
{
    if (rows == 0 || k == 0) return cudaSuccess;
    DeviceInfo dev;
    cudaError_t e = device_info(&dev);
    if (e != cudaSuccess) return e;
    // one warp per 2048 codes of a row, at most one wave of resident blocks
    // (every block gets the same share of a grid-stride loop, so a second,
    // partial wave would double the time of the blocks in it)
    const int64_t warps = rows * ((k + 2047) / 2048);
    int64_t grid = (warps + kThreads / 32 - 1) / (kThreads / 32);
    const int64_t cap = (int64_t)dev.sm_count * dequantize_blocks_per_sm(fmt);
    if (grid > cap) grid = cap;
    if (fmt == kNv)
        dequantize_kernel<kNv><<<(unsigned)grid, kThreads, 0, s>>>(packed, scales, gs, rows, k, out, ld);
    else if (fmt == kP1)
        dequantize_kernel<kP1><<<(unsigned)grid, kThreads, 0, s>>>(packed, scales, gs, rows, k, out, ld);
    else
        dequantize_kernel<kMx><<<(unsigned)grid, kThreads, 0, s>>>(packed, scales, gs, rows, k, out, ld);
    return cudaGetLastError();
}

cudaError_t launch_quantize(int fmt, int axis, const uint16_t* x, int64_t rows, int64_t cols,
                            int64_t ld, uint8_t* packed, uint8_t* scales, const float* gs,
                            cudaStream_t s)
{
    if (rows == 0 || cols == 0) return cudaSuccess;
    const int kb = block_size(fmt);
    if (axis == 0) {
        const RowwiseDesc d = {x, rows, cols, ld, packed, scales, gs};
        return launch_quantize_rowwise_batch(fmt, 1, &d, s);
    } else {
        dim3 grid((unsigned)(rows / (4 * kb)), (unsigned)((cols + 127) / 128));
        if (fmt == kNv)
            quantize_colwise_kernel<kNv><<<grid, kThreads, 0, s>>>(x, rows, cols, ld, packed, scales, gs);
        else if (fmt == kP1)
            quantize_colwise_kernel<kP1><<<grid, kThreads, 0, s>>>(x, rows, cols, ld, packed, scales, gs);
        else
            quantize_colwise_kernel<kMx><<<grid, kThreads, 0, s>>>(x, rows, cols, ld, packed, scales, gs);
    }
    return cudaGetLastError();
}

}  // namespace fp4
