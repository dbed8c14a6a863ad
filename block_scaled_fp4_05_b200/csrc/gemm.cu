// W4A4 block-scaled GEMM on the 5th-generation tensor cores (sm_100a):
// D = alpha * A_hat * B_hat^T, A_hat/B_hat = E2M1 codes times per-block scales.
//
// Method: "NVFP4 Architecture: Microscaling & 4-Bit LLMs on Blackwell",
// "2. Hardware-Managed Tensor Core Dot-Products" (TMA streams the packed
// 4-bit tiles and their scale vectors into shared memory; the tensor core
// forms the block dot products, multiplies them by S_u * S_v and accumulates
// in FP32) and "How Microscaling FP4 (MXFP4) Halves Memory Bandwidth...",
// "Silicon Execution" (accumulate in 32-bit precision before storing).
//
// Two kernels: fp4_gemm_pair_kernel (prefill and grouped problems, CTA pairs,
// described before its definition) and fp4_gemm_kernel (one CTA per tile,
// used in the decode form).  Structure of the latter, which the pair kernel
// shares role for role (one CTA per SM, persistent):
//   warp 0      TMA producer: packed A/B tiles via tensor maps (128-byte
//               swizzle), scale chunks via 1-D bulk copies, into a ring of
//               STAGES shared-memory stages guarded by full/empty mbarriers.
//   warp 1      TMEM allocation; one thread issues tcgen05.mma
//               (kind::mxf4nvf4, block_scale, 128 x BN x 64 per instruction)
//               and tcgen05.commit to release stages and to publish the
//               accumulator.
//   warps 2-5   epilogue: tcgen05.ld of the FP32 accumulator (each warp its
//               32-lane quadrant), alpha, BF16 round-to-nearest-even into
//               registers, release of the accumulator, then 16-byte stores;
//               or FP32 split-K partials (decode form).
//   warps 6-9   scale staging: each warp copies the stage's scale chunks from
//               shared memory into its own TMEM lane quadrant with
//               tcgen05.st, so that the tensor pipe only runs MMAs (a
//               tcgen05.cp of a 512-byte chunk occupies the tensor pipe for
//               about half the time of a 128x256x64 MMA).
//   warps 10-13 (the decode tile, N = 16, only) when the activation arrives
//               as BF16: each forms the NVFP4 codes and scales of every
//               fourth stage's activation slice straight into that stage's
//               shared-memory slot (otherwise they idle).
// Every mbarrier wait is bounded by %globaltimer; on expiry the CTA sets the
// library's device error word, stops issuing work, drains what it already
// issued, frees its tensor memory and returns (no trap).
//
// Scale layout in tensor memory: one 512-byte chunk (128 rows x 4 scale
// bytes, the global tile layout) occupies 4 TMEM columns; in every lane
// quadrant, column c, lane l holds the 4 scale bytes of row 32c + l (lane l
// of each staging warp writes the chunk's 16-byte row l).  For NVFP4
// (scale_vec::4X, E4M3) one chunk serves one K=64 MMA; for MXFP4
// (scale_vec::2X, E8M0) one chunk serves two, selected by scale-factor id 0/2.
//
// Decode form (M <= 16 tokens): the operands are swapped so that the weight
// rows fill the 128-row MMA side and the tokens form a 16-wide N side.  The
// weight tiles are scheduled as stream-K followed by data-parallel tiles: the
// (weight tile, K stage) units of the first sk_tiles tiles are split evenly
// over the CTAs, each CTA writes FP32 partials per such tile it touched, and
// the CTA that completes a tile sums its partials in a fixed (CTA) order,
// applies alpha and writes BF16; then every CTA runs whole tiles, written
// straight from the accumulator.  The split-K reductions thus overlap the
// whole-tile phase instead of trailing the kernel.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "fp4_internal.h"
#include "quant_device.cuh"

namespace fp4 {

__device__ unsigned int g_fp4_error_word;

namespace {

constexpr int BM = 128;             // MMA M (rows of the A-side operand per tile)
constexpr int BK = 256;             // K elements per pipeline stage (128 bytes/row)
constexpr int BK_BYTES = BK / 2;
constexpr int MMA_K = 64;           // K per tcgen05.mma for FP4
constexpr int A_BYTES = BM * BK_BYTES;
constexpr int SF_CHUNK = 512;       // 128 rows x 4 scale bytes
constexpr int SFA_BYTES = 4 * SF_CHUNK;
// 10 warps: producer, MMA, 4 epilogue, 4 scale staging; the decode tile
// (N = 16) adds 4 activation-quantizer warps
template <int BN>
constexpr int kThreadsFor = BN == 16 ? 448 : 320;
constexpr uint64_t kTimeoutNs = 2000000000ull;

enum : unsigned { ERR_FULL = 1u, ERR_EMPTY = 2u, ERR_ACC_FULL = 4u, ERR_ACC_EMPTY = 8u,
                  ERR_DRAIN = 16u, ERR_SELFTEST = 32u, ERR_WORKSPACE = kErrorWorkspaceBit };

template <int BN, int STAGES>
struct Cfg {
    static constexpr int BH = (BN + 127) / 128;          // 128-row scale tiles of B per tile
    static constexpr int B_BYTES = BN * BK_BYTES;
    static constexpr int SFB_BYTES = BH * SFA_BYTES;
    static constexpr int STAGE_RAW = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int STAGE_BYTES = (STAGE_RAW + 1023) / 1024 * 1024;
    static constexpr int OFF_B = A_BYTES;
    static constexpr int OFF_SFA = A_BYTES + B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + SFA_BYTES;
    static constexpr int SF_COL0 = BN < 32 ? 32 : BN;    // first TMEM column of the scale ring
    static constexpr int SFA_COLS = 4 * 4;               // 4 chunks x 4 columns
    static constexpr int SF_COLS = SFA_COLS + 4 * 4 * BH;
    static constexpr int TMEM_COLS = 512;
    // barriers (1 KB), then, for the decode tile, the activation scale bytes
    // of each stage formed in the kernel (16 rows x 16 bytes per stage)
    static constexpr int OFF_ACT = 1024;   // from the barrier area
    static constexpr int ACT_SF_BYTES = BN == 16 ? STAGES * 256 : 0;
    static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + OFF_ACT + ACT_SF_BYTES;
    static_assert(SF_COL0 + STAGES * SF_COLS <= TMEM_COLS, "tensor memory overflow");
    static_assert(SMEM <= 232448, "shared memory per block");
    static_assert(BN % 16 == 0 && BN <= 256, "MMA N");
    static_assert(BH <= 2, "scale staging covers at most two 128-row tiles of B");
    static_assert((3 * STAGES + 3) * 8 + 8 <= 40 * 8, "barrier area below the activation barriers");
    static_assert((40 + STAGES) * 8 <= OFF_ACT, "activation barriers below the scale buffers");
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms stay 1024-aligned");
};

struct Params {
    const uint8_t* sfa;
    const uint8_t* sfb;
    int32_t rows_a, rows_b, K;
    int32_t ks_total;          // K stages per tile
    int32_t sf_col_tiles;      // 512-byte scale tiles per 128-row group
    int32_t sfa_row_tiles, sfb_row_tiles;
    int32_t tiles_m, tiles_n;
    int32_t units;             // stream-K: sk_tiles * ks_total
    int32_t sk_tiles;          // stream-K: tiles split over the CTAs; the rest run whole
    int32_t a_static;          // A side not written by the previous kernel: prefetch it
    int32_t raster_gm;         // pair kernel: M tiles per group of the tile order
    int32_t max_seg;           // stream-K: partial slots per CTA
    const float* alpha;
    uint16_t* D;
    int64_t ldd;
    float* ws;
    int* counters;             // stream-K: arrivals per (weight tile, lane quadrant)
    // decode form with the activation quantized in the kernel (else NULL):
    // BF16 activation [rows_b x K] with leading dimension lda, and its
    // S_global (written by the kernel before this one)
    const uint16_t* act;
    int64_t lda;
    const float* act_gs;
};

// ------------------------------------------------------------------------
// PTX wrappers
// ------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t now_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of `bar` with the given parity.  Gives up when another
// role has raised the CTA's abort flag or after kTimeoutNs; in the latter
// case raises the flag and records `code` in the device error word.
__device__ __noinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned code)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = now_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 0) {
            if (*abort_flag) return false;
            if (now_ns() - t0 > kTimeoutNs) {
                *abort_flag = 1;
                atomicOr(&g_fp4_error_word, code);
                return false;
            }
        }
    }
}

// Inline fast path: one try_wait, the bounded loop only when it fails.
__device__ __forceinline__ bool wait_fast(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned code)
{
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bounded(bar, parity, abort_flag, code);
}

// Wait that ignores the abort flag (used only to drain work already issued).
__device__ __noinline__ bool wait_drain(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = now_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (now_ns() - t0 > kTimeoutNs) {
            atomicOr(&g_fp4_error_word, ERR_DRAIN);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint32_t bar, uint32_t dst,
                                            int32_t x, int32_t y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Device-scope release-acquire atomic increment (returns the old value).
__device__ __forceinline__ int atomic_add_acq_rel(int* p, int v)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Programmatic dependent launch.  The GEMM kernels are launched so that they
// may start while the kernel before them on the stream is still running;
// pdl_wait() blocks until that kernel has completed and its writes are
// visible, and every thread that reads an operand, the scales or alpha, or
// writes D or the workspace, passes it first.  Everything before it (barrier
// set-up, tensor memory allocation, tensor-map prefetch) overlaps the
// previous kernel.  Without the launch attribute it returns at once.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next kernel on the stream (if launched with the attribute) begin.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

template <bool MX>
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    if (MX) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::2X"
            " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X"
            " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
            : "memory");
    }
}

// Shared-memory matrix descriptor: K-major rows of 128 bytes with the
// 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::mxf4nvf4 with block scaling: E2M1 x E2M1,
// FP32 accumulate, K-major A and B, M = 128, N = BN; scale type UE8M0
// (MXFP4, and 16-element blocks with E8M0 scales) or UE4M3 (NVFP4); sf_id
// selects the scale byte pair (2X) inside each column.
template <int BN, int FMT>
__device__ __forceinline__ uint32_t make_idesc(uint32_t sf_id)
{
    return (sf_id << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
           ((FMT != kNv ? 1u : 0u) << 23) | ((uint32_t)(BM >> 4) << 24) | (sf_id << 29);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32"
        " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Completes outstanding tcgen05.ld; the registers are threaded through so
// that no use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[16])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32"
        " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                   "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7])
                 : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32"
        " [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32"
        " [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ------------------------------------------------------------------------
// Work schedule shared by the three roles.  A segment is a run of K stages
// of one output tile.
// ------------------------------------------------------------------------
struct Seg {
    int tm, tn, kb, ke, slot;
};
// In the decode schedule a segment that covers a whole tile has no other
// contributor and is written straight to D.

template <bool STREAM_K>
struct Schedule {
    const Params& p;
    int next_tile;   // prefill: next tile index; decode: next whole tile
    int u, ue, ub;   // stream-K: unit cursor / range
    __device__ explicit Schedule(const Params& pp) : p(pp)
    {
        if (STREAM_K) {
            const int64_t G = gridDim.x;
            ub = (int)(((int64_t)blockIdx.x * p.units) / G);
            ue = (int)(((int64_t)(blockIdx.x + 1) * p.units) / G);
            u = ub;
            next_tile = p.sk_tiles + blockIdx.x;
        } else {
            next_tile = blockIdx.x;
        }
    }
    __device__ bool next(Seg& s)
    {
        if (STREAM_K) {
            s.tn = 0;
            if (u < ue) {
                s.tm = u / p.ks_total;
                s.kb = u % p.ks_total;
                const int left = ue - u;
                s.ke = min(p.ks_total, s.kb + left);
                s.slot = s.tm - ub / p.ks_total;
                u += s.ke - s.kb;
                return true;
            }
            if (next_tile >= p.tiles_m) return false;
            s.tm = next_tile;
            s.kb = 0;
            s.ke = p.ks_total;
            s.slot = 0;
            next_tile += gridDim.x;
            return true;
        } else {
            if (next_tile >= p.tiles_m * p.tiles_n) return false;
            s.tm = next_tile % p.tiles_m;
            s.tn = next_tile / p.tiles_m;
            s.kb = 0;
            s.ke = p.ks_total;
            s.slot = 0;
            next_tile += gridDim.x;
            return true;
        }
    }
};

// ------------------------------------------------------------------------
// The kernel
// ------------------------------------------------------------------------
template <int BN, int STAGES, int FMT, bool STREAM_K>
__global__ void __launch_bounds__(kThreadsFor<BN>, 1)
fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const Params p)
{
    constexpr bool MX = FMT == kMx;   // 32-element blocks (scale_vec::2X); else 16 (4X)
    using C = Cfg<BN, STAGES>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
    // bars[0..S): full, [S..2S): empty, [2S..3S): scales staged,
    // [3S]: acc_full, [3S+1]: acc_empty, [3S+2]: drain
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * STAGES + 3);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t smem0 = smem_u32(smem);
    auto full = [&](int s) { return smem_u32(&bars[s]); };
    auto empty = [&](int s) { return smem_u32(&bars[STAGES + s]); };
    auto sf_ready = [&](int s) { return smem_u32(&bars[2 * STAGES + s]); };
    auto act_full = [&](int s) { return smem_u32(&bars[40 + s]); };
    const uint32_t acc_full = smem_u32(&bars[3 * STAGES]);
    const uint32_t acc_empty = smem_u32(&bars[3 * STAGES + 1]);
    const uint32_t drain = smem_u32(&bars[3 * STAGES + 2]);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
            mbar_init(sf_ready(s), 4);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 4);
        mbar_init(drain, 1);
        // activation stage published by a quantizer warp (in-kernel
        // activation quantization, decode tile)
        for (int s = 0; s < STAGES; ++s) mbar_init(smem_u32(&bars[40 + s]), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
            const uint32_t bar0 = smem_u32(bars);
            const int64_t sf_row_bytes = (int64_t)p.sf_col_tiles * SF_CHUNK;
            // scale row tiles of B that exist for a tile
            auto count_nbh = [&](const Seg& g) {
                const int rtb0 = (g.tn * BN) / 128;
                int nbh = 0;
                for (int h = 0; h < C::BH; ++h)
                    if (rtb0 + h < p.sfb_row_tiles) ++nbh;
                return nbh;
            };
            // Requests the A side (A tile + its scales) and/or the B side of
            // K stage ks of segment g into ring slot stg; `expect` posts the
            // stage's full byte count on its barrier.
            auto issue = [&](int stg, const Seg& g, int ks, int nbh, bool a_side, bool b_side, bool expect) {
                // (b_side is cleared below for an activation quantized in the kernel)
                const uint32_t fb = bar0 + 8u * stg;
                const int nk = min(4, (p.K - ks * BK) / MMA_K);
                const int nch = MX ? nk / 2 : nk;
                const int ct0 = MX ? ks * 2 : ks * 4;   // first 512-byte scale chunk of the stage
                const uint32_t sf_bytes = (uint32_t)nch * SF_CHUNK;
                const uint32_t st = smem0 + stg * C::STAGE_BYTES;
                const bool dyn = !MX && BN == 16 && p.act != nullptr;   // activation quantized by the staging warps
                if (expect)
                    mbar_arrive_expect_tx(fb, dyn ? A_BYTES + sf_bytes
                                                  : A_BYTES + C::B_BYTES + sf_bytes * (1 + nbh));
                if (dyn) b_side = false;
                if (a_side) {
                    tma_load_2d(&tmA, fb, st, ks * BK_BYTES, g.tm * BM);
                    bulk_load(st + C::OFF_SFA, p.sfa + g.tm * sf_row_bytes + ct0 * SF_CHUNK, sf_bytes, fb);
                }
                if (b_side) {
                    const uint8_t* sfb_row = p.sfb + ((g.tn * BN) / 128) * sf_row_bytes;
                    tma_load_2d(&tmB, fb, st + C::OFF_B, ks * BK_BYTES, g.tn * BN);
                    if (nbh > 0) bulk_load(st + C::OFF_SFB, sfb_row + ct0 * SF_CHUNK, sf_bytes, fb);
                    if (C::BH == 2 && nbh > 1)
                        bulk_load(st + C::OFF_SFB + SFA_BYTES, sfb_row + sf_row_bytes + ct0 * SF_CHUNK,
                                  sf_bytes, fb);
                }
            };
            // Static A side (the weights, in the decode form): the first
            // STAGES stages' A tiles and scales are requested before the
            // dependency wait, so they stream in while the previous kernel
            // finishes; their B sides follow after it.
            int pre_n = 0;
            if (STREAM_K && p.a_static) {
                Schedule<STREAM_K> pre(p);
                Seg g;
                while (pre_n < STAGES && pre.next(g)) {
                    const int nbh = count_nbh(g);
                    for (int ks = g.kb; ks < g.ke && pre_n < STAGES; ++ks, ++pre_n)
                        issue(pre_n, g, ks, nbh, true, false, true);
                }
            }
            pdl_wait();
            Schedule<STREAM_K> sched(p);
            Seg sg;
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            while (ok && sched.next(sg)) {
                const int nbh = count_nbh(sg);
                for (int ks = sg.kb; ks < sg.ke; ++ks) {
                    if (issued < pre_n) {
                        issue(stage, sg, ks, nbh, false, true, false);   // A side already requested
                    } else {
                        if (!wait_fast(bar0 + 8u * (STAGES + stage), phase ^ 1u, abort_flag, ERR_EMPTY)) {
                            ok = false;
                            break;
                        }
                        issue(stage, sg, ks, nbh, true, true, true);
                    }
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            pdl_trigger();
            // Drain: the last min(issued, STAGES) stages may still be in flight
            // if the consumers stopped early; wait for their transactions.
            if (!ok || *abort_flag) {
                const int n = issued < STAGES ? issued : STAGES;
                for (int i = 1; i <= n; ++i) {
                    int s = stage - i;
                    uint32_t ph = phase;
                    if (s < 0) {
                        s += STAGES;
                        ph ^= 1u;
                    }
                    wait_drain(full(s), ph);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        // The loop is kept short: a 128x256x64 MMA lasts 128 cycles, so the
        // per-stage bookkeeping of this single thread must stay well below
        // the 512 cycles of tensor work a 256-deep stage carries.
        if (lane == 0) {
            const uint32_t bar0 = smem_u32(bars);
            const uint64_t adesc0 = desc_sw128(smem0);
            const uint64_t bdesc0 = desc_sw128(smem0 + C::OFF_B);
            constexpr uint32_t kDescPerStage = C::STAGE_BYTES >> 4;   // start-address field step
            const uint32_t idesc0 = make_idesc<BN, FMT>(0);
            const uint32_t idesc2 = make_idesc<BN, FMT>(2);
            const uint32_t tsf0 = tmem_base + C::SF_COL0;
            Schedule<STREAM_K> sched(p);
            Seg sg;
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            while (ok && sched.next(sg)) {
                if (!wait_fast(acc_empty, acc_phase ^ 1u, abort_flag, ERR_ACC_EMPTY)) break;
                tc_fence_after();
                for (int ks = sg.kb; ks < sg.ke; ++ks) {
                    if (!wait_fast(bar0 + 8u * stage, phase, abort_flag, ERR_FULL) ||
                        !wait_fast(bar0 + 8u * (2 * STAGES + stage), phase, abort_flag, ERR_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = adesc0 + (uint64_t)(stage * kDescPerStage);
                    const uint64_t bd = bdesc0 + (uint64_t)(stage * kDescPerStage);
                    const uint32_t tsf = tsf0 + stage * C::SF_COLS;
                    const uint32_t tsfb = tsf + C::SFA_COLS;
                    const uint32_t acc0 = ks > sg.kb ? 1u : 0u;
                    const int nk = min(4, (p.K - ks * BK) / MMA_K);
                    if (nk == 4) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int chunk = MX ? (j >> 1) : j;
                            tc_mma<MX>(tmem_base, ad + 2 * j, bd + 2 * j,
                                       (MX && (j & 1)) ? idesc2 : idesc0, tsf + 4 * chunk,
                                       tsfb + chunk * C::BH * 4, j > 0 ? 1u : acc0);
                        }
                    } else {
                        for (int j = 0; j < nk; ++j) {
                            const int chunk = MX ? (j >> 1) : j;
                            tc_mma<MX>(tmem_base, ad + 2 * j, bd + 2 * j,
                                       (MX && (j & 1)) ? idesc2 : idesc0, tsf + 4 * chunk,
                                       tsfb + chunk * C::BH * 4, j > 0 ? 1u : acc0);
                        }
                    }
                    tc_commit(bar0 + 8u * (STAGES + stage));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(acc_full);
                acc_phase ^= 1u;
            }
            // make sure every tcgen05 operation issued here has completed
            tc_commit(drain);
            wait_drain(drain, 0);
        }
    } else if (warp < 6) {
        // ---------------- epilogue (warps 2..5) ----------------
        const int q = warp & 3;               // TMEM lane quadrant of this warp
        const int row = q * 32 + lane;        // accumulator row of this thread
        pdl_wait();
        const float alpha = p.alpha ? *p.alpha : 1.0f;
        const uint32_t trow = tmem_base + ((uint32_t)(q * 32) << 16);
        Schedule<STREAM_K> sched(p);
        Seg sg;
        uint32_t acc_phase = 0;
        while (sched.next(sg)) {
            // lane 0 polls, the warp follows it as a whole so that the
            // .sync.aligned tensor-memory loads below stay warp-uniform
            int ok = 0;
            if (lane == 0) ok = wait_bounded(acc_full, acc_phase, abort_flag, ERR_ACC_FULL) ? 1 : 0;
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) break;
            __syncwarp();
            tc_fence_after();
            if constexpr (!STREAM_K) {
                // whole row of the tile into registers as BF16 pairs, then
                // hand the accumulator back before the global stores
                uint32_t packed[BN / 2];
#pragma unroll
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(trow + c * 32, r);
                    tmem_wait_ld(r);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        packed[c * 16 + i] =
                            pack_bf16x2(__fmul_rn(alpha, __uint_as_float(r[2 * i])),
                                        __fmul_rn(alpha, __uint_as_float(r[2 * i + 1])));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty);
                const int64_t gm = (int64_t)sg.tm * BM + row;
                if (gm < p.rows_a) {
                    uint16_t* drow = p.D + gm * p.ldd + (int64_t)sg.tn * BN;
                    const int ncols = p.rows_b - sg.tn * BN;
#pragma unroll
                    for (int i = 0; i < BN / 8; ++i)
                        if (i * 8 < ncols)
                            *reinterpret_cast<uint4*>(drow + i * 8) =
                                make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2],
                                           packed[4 * i + 3]);
                }
            } else {
                static_assert(BN == 16, "the stream-K epilogue reads one 16-column chunk");
                uint32_t r[16];
                tmem_ld16(trow, r);
                tmem_wait_ld(r);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty);
                if (sg.kb == 0 && sg.ke == p.ks_total) {
                    // whole tile: no other contributor
                    const int64_t n = (int64_t)sg.tm * BM + row;
                    if (n < p.rows_a) {
#pragma unroll
                        for (int m = 0; m < 16; ++m)
                            if (m < p.rows_b) {
                                const uint32_t b = pack_bf16x2(__fmul_rn(alpha, __uint_as_float(r[m])), 0.0f);
                                p.D[(int64_t)m * p.ldd + n] = (uint16_t)(b & 0xFFFFu);
                            }
                    }
                    acc_phase ^= 1u;
                    continue;
                }
                // FP32 partial of this segment; the CTA whose partial completes
                // a weight tile (per 32-row lane quadrant) sums all partials of
                // that tile in CTA order and writes the BF16 outputs.  Ordering
                // (the usual semaphore pattern): every lane's partial stores,
                // a device-scope fence by every lane, a warp barrier, then lane
                // 0's release-acquire increment; in the last arriver, lane 0's
                // acquire, a warp barrier and a fence by every lane before the
                // other partials are read.
                float* slot = p.ws + ((int64_t)blockIdx.x * p.max_seg + sg.slot) * (BN * BM);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (j < p.rows_b) __stcg(slot + j * BM + row, __uint_as_float(r[j]));
                __threadfence();
                __syncwarp();
                const int64_t G = gridDim.x;
                const int64_t x0 = (int64_t)sg.tm * p.ks_total, x1 = x0 + p.ks_total - 1;
                const int c0 = (int)(((x0 + 1) * G - 1) / p.units);
                const int c1 = (int)(((x1 + 1) * G - 1) / p.units);
                int* counter = p.counters + sg.tm * 4 + q;
                int last = 0;
                if (lane == 0) {
                    const int old = atomic_add_acq_rel(counter, 1);
                    last = old == c1 - c0 ? 1 : 0;
                    if (old < 0 || old > c1 - c0) atomicOr(&g_fp4_error_word, ERR_WORKSPACE);
                }
                last = __shfl_sync(0xFFFFFFFFu, last, 0);
                if (last) {
                    __syncwarp();
                    __threadfence();
                    const int64_t n = (int64_t)sg.tm * BM + row;
                    float sum[16];
#pragma unroll
                    for (int m = 0; m < 16; ++m) sum[m] = 0.0f;
                    // contributors in CTA order, up to four partial rows in
                    // flight at a time; this CTA's own values come from registers
                    for (int cb = c0; cb <= c1; cb += 4) {
                        float v[4][16];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int c = cb + i;
                            if (c > c1) break;
                            if (c == (int)blockIdx.x) {
#pragma unroll
                                for (int m = 0; m < 16; ++m) v[i][m] = __uint_as_float(r[m]);
                                continue;
                            }
                            const int ubc = (int)(((int64_t)c * p.units) / G);
                            const int slot_c = sg.tm - ubc / p.ks_total;
                            const float* part = p.ws + ((int64_t)c * p.max_seg + slot_c) * (BN * BM) + row;
#pragma unroll
                            for (int m = 0; m < 16; ++m) v[i][m] = m < p.rows_b ? __ldcg(part + m * BM) : 0.0f;
                        }
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            if (cb + i > c1) break;
#pragma unroll
                            for (int m = 0; m < 16; ++m) sum[m] = __fadd_rn(sum[m], v[i][m]);
                        }
                    }
                    if (n < p.rows_a) {
#pragma unroll
                        for (int m = 0; m < 16; ++m)
                            if (m < p.rows_b) {
                                const uint32_t b = pack_bf16x2(__fmul_rn(alpha, sum[m]), 0.0f);
                                p.D[(int64_t)m * p.ldd + n] = (uint16_t)(b & 0xFFFFu);
                            }
                    }
                    if (lane == 0) *counter = 0;   // ready for the next call
                }
            }
            acc_phase ^= 1u;
        }
    } else if (warp < 10) {
        // ---------------- scale staging (warps 6..9) ----------------
        // Each warp writes its own TMEM lane quadrant: lane l stores the
        // 16-byte row l of every 512-byte chunk (4 consecutive columns).
        // With an activation quantized in the kernel (decode form, p.act set)
        // the activation's scale bytes come from the quantizer warps'
        // per-stage buffer (16 rows x 16 bytes) once act_full[stage] is set.
        const uint32_t tq = tmem_base + ((uint32_t)((warp & 3) * 32) << 16);
        const bool dyn = !MX && BN == 16 && p.act != nullptr;
        const uint8_t* act_sf = reinterpret_cast<const uint8_t*>(bars) + C::OFF_ACT;
        Schedule<STREAM_K> sched(p);
        Seg sg;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        while (ok && sched.next(sg)) {
            const int rtb0 = (sg.tn * BN) / 128;
            int nbh = 0;
            for (int h = 0; h < C::BH; ++h)
                if (rtb0 + h < p.sfb_row_tiles) ++nbh;
            for (int ks = sg.kb; ks < sg.ke; ++ks) {
                int w = 0;
                if (lane == 0) {
                    w = wait_bounded(full(stage), phase, abort_flag, ERR_FULL) ? 1 : 0;
                    if (w && dyn) w = wait_fast(act_full(stage), phase, abort_flag, ERR_FULL) ? 1 : 0;
                }
                w = __shfl_sync(0xFFFFFFFFu, w, 0);
                if (!w) {
                    ok = false;
                    break;
                }
                __syncwarp();
                tc_fence_after();
                const int nk = min(4, (p.K - ks * BK) / MMA_K);
                const int nch = MX ? nk / 2 : nk;
                const uint32_t st = smem0 + stage * C::STAGE_BYTES + lane * 16;
                const uint32_t tsf = tq + C::SF_COL0 + stage * C::SF_COLS;
                uint32_t a[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (j < nch) v = ld_shared_v4(st + C::OFF_SFA + j * SF_CHUNK);
                    a[4 * j] = v.x;
                    a[4 * j + 1] = v.y;
                    a[4 * j + 2] = v.z;
                    a[4 * j + 3] = v.w;
                }
                tmem_st16(tsf, a);
                if constexpr (C::BH == 2) {
                    uint32_t b[32];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            uint4 v = make_uint4(0u, 0u, 0u, 0u);
                            if (j < nch && h < nbh)
                                v = ld_shared_v4(st + C::OFF_SFB + h * SFA_BYTES + j * SF_CHUNK);
                            b[(j * 2 + h) * 4] = v.x;
                            b[(j * 2 + h) * 4 + 1] = v.y;
                            b[(j * 2 + h) * 4 + 2] = v.z;
                            b[(j * 2 + h) * 4 + 3] = v.w;
                        }
                    tmem_st32(tsf + C::SFA_COLS, b);
                } else {
                    uint32_t b[16];
                    if (dyn) {
                        // lane l < 16 holds activation row l: its word j carries
                        // blocks 4j..4j+3; the other rows of the chunk are padding
                        uint4 v = make_uint4(0u, 0u, 0u, 0u);
                        if (lane < 16) v = *reinterpret_cast<const uint4*>(act_sf + stage * 256 + lane * 16);
                        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            b[4 * j] = j < nch ? wv[j] : 0u;
                            b[4 * j + 1] = 0u;
                            b[4 * j + 2] = 0u;
                            b[4 * j + 3] = 0u;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint4 v = make_uint4(0u, 0u, 0u, 0u);
                            if (j < nch && nbh > 0) v = ld_shared_v4(st + C::OFF_SFB + j * SF_CHUNK);
                            b[4 * j] = v.x;
                            b[4 * j + 1] = v.y;
                            b[4 * j + 2] = v.z;
                            b[4 * j + 3] = v.w;
                        }
                    }
                    tmem_st16(tsf + C::SFA_COLS, b);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sf_ready(stage));
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if constexpr (!MX && BN == 16) {
        // ---------------- activation quantizer (warps 10..13, decode tile) ----------------
        // With p.act set, warp q = warp - 10 forms the activation operand of
        // the CTA's stages n = q, q + 4, q + 8, ...: the stage's 16 rows x 256
        // elements, lane l taking the 32-element chunk c = l % 8 (two
        // 16-element blocks) of rows l / 8 + 4 j, j = 0..3, quantized exactly
        // as fp4_quantize does (zero codes and scales outside the matrix).
        // The 16 code bytes of (row r, chunk c) go to the stage's B slot in
        // the 128-byte-swizzled layout a TMA load would have produced (16-byte
        // position c ^ (r % 8) of row r), the two scale bytes to the stage's
        // scale buffer (row r, bytes 2c, 2c + 1).  The loads and the
        // arithmetic run before the slot is free; the stores wait for the
        // MMA of the slot's previous use (the producer's empty barrier), and
        // the stage is published on act_full[stage].  Four warps take turns,
        // so the quantization of one stage overlaps that of the next three.
        if (p.act != nullptr) {
            pdl_wait();
            const float gs = *p.act_gs;
            const float denom = __fmul_rn(6.0f, gs);
            const int q = warp - 10;
            const int c = lane & 7;
            uint8_t* act_sf = reinterpret_cast<uint8_t*>(bars) + C::OFF_ACT;
            Schedule<STREAM_K> sched(p);
            Seg sg;
            int n = 0;
            bool ok = true;
            while (ok && sched.next(sg)) {
                for (int ks = sg.kb; ks < sg.ke; ++ks, ++n) {
                    if ((n & 3) != q) continue;
                    const int stage = n % STAGES;
                    const uint32_t phase = (uint32_t)(n / STAGES) & 1u;
                    const int k0 = ks * BK;
                    const int nk = min(4, (p.K - k0) / MMA_K);
                    uint4 v[4][4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int r = (lane >> 3) + 4 * j;
                        const bool in = r < p.rows_b && c < 2 * nk;
                        const uint4* src =
                            reinterpret_cast<const uint4*>(p.act + (int64_t)(in ? r : 0) * p.lda + k0 + (in ? c * 32 : 0));
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            v[j][u] = in ? qdev::ld_stream(src + u) : make_uint4(0u, 0u, 0u, 0u);
                    }
                    uint4 codes[4];
                    uint32_t sbw[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        float inv0, inv1;
                        const uint32_t s0 = qdev::block_scale<FMT>(
                            max(qdev::absmax8(v[j][0]), qdev::absmax8(v[j][1])), gs, denom, &inv0);
                        const uint32_t s1 = qdev::block_scale<FMT>(
                            max(qdev::absmax8(v[j][2]), qdev::absmax8(v[j][3])), gs, denom, &inv1);
                        codes[j] = make_uint4(qdev::quantize8(v[j][0], inv0), qdev::quantize8(v[j][1], inv0),
                                              qdev::quantize8(v[j][2], inv1), qdev::quantize8(v[j][3], inv1));
                        sbw[j] = s0 | (s1 << 8);
                    }
                    int w = 0;
                    if (lane == 0) w = wait_bounded(empty(stage), phase ^ 1u, abort_flag, ERR_EMPTY) ? 1 : 0;
                    w = __shfl_sync(0xFFFFFFFFu, w, 0);
                    if (!w) {
                        ok = false;
                        break;
                    }
                    __syncwarp();
                    const uint32_t slot = smem0 + stage * C::STAGE_BYTES + C::OFF_B;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int r = (lane >> 3) + 4 * j;
                        const uint32_t dst = slot + r * BK_BYTES + ((uint32_t)(c ^ (r & 7)) << 4);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(codes[j].x),
                                     "r"(codes[j].y), "r"(codes[j].z), "r"(codes[j].w)
                                     : "memory");
                        *reinterpret_cast<uint16_t*>(act_sf + stage * 256 + r * 16 + c * 2) = (uint16_t)sbw[j];
                    }
                    // the codes are read by the tensor core (async proxy)
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(act_full(stage));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(C::TMEM_COLS)
                     : "memory");
    }
}

// ------------------------------------------------------------------------
// CTA-pair kernel (prefill).  A cluster of two CTAs on neighbouring SMs
// computes a 256 x 256 tile with tcgen05.mma.cta_group::2: each CTA stages
// its own 128 rows of A and its half (128 rows) of the 256-row B tile, so a
// CTA moves 32 KB of operands per 256-deep stage instead of 48 KB for the
// same tensor work.  Each CTA keeps the scales of its own A rows and of all
// 256 B rows in its own TMEM and accumulates its 128 x 256 half of the tile
// there.
//   warp 0        producer: lane 0 runs the stage loop and issues the
//                 tensor loads of A and B (both CTAs' loads
//                 complete on the leader's (rank 0) full[s]; the leader posts
//                 the expected bytes of both) and the scale chunks (on the
//                 CTA's own sf_full[s]).
//   warp 1        MMA issue (leader CTA only): passes the stage's named
//                 barrier, then lane 0 issues the pair MMAs and releases the
//                 stage in both CTAs (and, after a tile, publishes the
//                 accumulator to both) with one commit that arrives on the
//                 barrier at the same offset in each CTA.  It waits on no
//                 mbarrier inside the loop.
//   warp 14       gatekeeper (leader CTA only): waits on the accumulator's
//                 release and on each stage's full barrier, then lets the
//                 MMA warp through the stage's named barrier (1 + stage).
//   warps 2-5, 10-13  epilogue: two warps per TMEM lane quadrant, each
//                 draining 128 of the 256 accumulator columns (tcgen05.ld,
//                 alpha, BF16), releasing the accumulator on the leader's
//                 acc_empty, then storing D through shared memory with TMA.
//   warps 6-9     scale staging: copy the stage's scale chunks into their
//                 TMEM lane quadrant with tcgen05.st, then arrive on the
//                 leader's full[s], so that full[s] completes when the
//                 operands of both CTAs have landed and both CTAs' scales are
//                 in TMEM.
// In the producer warp the other 31 lanes wait at __syncwarp (not at a
// warp-aligned barrier) while lane 0 runs the loop; the MMA warp runs the
// loop with all lanes (the named barrier takes whole warps), lane 0 issuing.
// All waits are bounded; a CTA that gives up records the error, and both
// CTAs meet at a final cluster barrier before the pair frees its TMEM.
// ------------------------------------------------------------------------
constexpr int PAIR_BN = 256;                 // N of the pair tile
constexpr int64_t kRasterGroupBytes = int64_t(32) << 20;   // A bytes per raster group
constexpr int PAIR_BHALF = PAIR_BN / 2;      // B rows staged by each CTA
constexpr int kPairThreads = 480;            // 15 warps, roles above
constexpr int kGateWarp = 14;                // the gatekeeper warp of the pair kernel
constexpr int kEpiWarps = 8;

// Per stage, NVFP4 carries 4 scale chunks per 128 rows (one per K=64 MMA),
// MXFP4 2 (one per two MMAs).
template <int STAGES, bool MX>
struct PairCfg {
    static constexpr int NCH = MX ? 2 : 4;                          // scale chunks per 128 rows
    static constexpr int B_BYTES = PAIR_BHALF * BK_BYTES;           // 16 KB
    static constexpr int SFA_STAGE = NCH * SF_CHUNK;
    static constexpr int SFB_STAGE = 2 * NCH * SF_CHUNK;            // 256 B rows: 2 row tiles
    static constexpr int STAGE_RAW = A_BYTES + B_BYTES + SFA_STAGE + SFB_STAGE;
    static constexpr int STAGE_BYTES = (STAGE_RAW + 1023) / 1024 * 1024;
    static constexpr int OFF_B = A_BYTES;
    static constexpr int OFF_SFA = A_BYTES + B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + SFA_STAGE;
    static constexpr int SF_COL0 = PAIR_BN;                        // accumulator: columns [0, 256)
    static constexpr int SFA_COLS = 4 * NCH;
    static constexpr int SF_COLS = SFA_COLS + 8 * NCH;
    static constexpr int TMEM_COLS = 512;
    static constexpr int NBARS = 3 * STAGES + 3;
    // arrivals that complete full[s] on the leader: the producer's
    // expect-tx arrival and the 4 scale-staging warps of each CTA
    static constexpr int FULL_ARRIVALS = 1 + 8;
    // epilogue staging: per epilogue warp one 32-row x 32-column BF16 block
    // (64-byte rows, 64-byte swizzle) that a TMA store writes to D
    static constexpr int EPI_BLOCK = 32 * 64;
    static constexpr int OFF_EPI = STAGES * STAGE_BYTES;
    static constexpr int OFF_BARS = OFF_EPI + kEpiWarps * EPI_BLOCK;
    static constexpr int SMEM = OFF_BARS + 1024 + 512;
    static_assert(SF_COL0 + STAGES * SF_COLS <= TMEM_COLS, "tensor memory overflow");
    static_assert(NBARS * 8 + 8 <= 512, "barrier area");
    static_assert(SMEM <= 232448, "shared memory per CTA");
    static_assert(STAGES + 1 <= 16, "one named barrier per stage (ids 1..STAGES)");
};

// 2-D TMA store of a shared-memory box to global memory (bulk-group
// completion), and the waits on this thread's bulk groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(x), "r"(y)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Hardware named barrier `id` of `count` threads: wait (all lanes of the
// calling warp) / arrive without waiting.
__device__ __forceinline__ void named_bar_sync(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void named_bar_arrive(int id, int count)
{
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// Arrive on a barrier of the other CTA without a cluster-scope release
// fence.  Used only after tcgen05.wait::st / wait::ld, which already
// guarantee that the tensor-memory accesses the arrival announces have
// completed; the cluster-scope release would cost ~1000 cycles per arrival.
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

// 2-D tensor load whose completion is counted on a barrier of either CTA of
// the pair (here: the leader's), destination in the issuing CTA.
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap* map, uint32_t bar_cluster,
                                                 uint32_t dst, int32_t x, int32_t y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
        : "memory");
}

// Arrive on the barrier at offset `bar` in both CTAs of the pair once the
// pair MMAs issued so far (by this thread) have completed.
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(bar),
        "h"((uint16_t)3)
        : "memory");
}

template <bool MX>
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                            uint32_t accumulate)
{
    if (MX) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::2X"
            " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X"
            " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
            : "memory");
    }
}

// Instruction descriptor of the pair MMA: M = 256 (128 rows per CTA), N = 256
// (or 128 for a half tile).
template <int FMT>
__device__ __forceinline__ uint32_t make_idesc_pair(uint32_t sf_id, uint32_t n = PAIR_BN)
{
    return (sf_id << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) |
           ((FMT != kNv ? 1u : 0u) << 23) | ((uint32_t)(256 >> 4) << 24) | (sf_id << 29);
}

__device__ __forceinline__ void spin_ns(uint64_t ns)
{
    const uint64_t t0 = now_ns();
    while (now_ns() - t0 < ns) {
    }
}

// Warp-uniform bounded wait, called by all 32 lanes of a warp: every lane
// polls and the warp leaves together.  Gives up (false) when the CTA's abort
// flag is raised or after kTimeoutNs, in which case it raises the flag and
// records `code` in the device error word.
__device__ __noinline__ bool warp_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                            unsigned code)
{
    const uint64_t t0 = now_ns();
    for (uint32_t it = 1;; ++it) {
        if (__all_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity))) return true;
        if ((it & 15u) == 0) {
            int give_up = 0;
            if ((threadIdx.x & 31) == 0) {
                if (*abort_flag) {
                    give_up = 1;
                } else if (now_ns() - t0 > kTimeoutNs) {
                    *abort_flag = 1;
                    atomicOr(&g_fp4_error_word, code);
                    give_up = 1;
                }
            }
            if (__shfl_sync(0xFFFFFFFFu, give_up, 0)) return false;
        }
    }
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned code)
{
    if (__all_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity))) return true;
    return warp_wait_slow(bar, parity, abort_flag, code);
}

// The problems one pair-kernel launch computes: NG = 1 for fp4_gemm, up to
// kMaxGroups for fp4_gemm_grouped.  Tile t of the launch belongs to problem g
// with tile_begin[g] <= t < tile_begin[g + 1]; within a problem, M tiles
// run fastest.
constexpr int kMaxGroups = 16;

template <int NG>
struct PairArgs {
    CUtensorMap a[NG], b[NG], d[NG];   // A, B (K-major, 128-byte swizzle) and D of each problem
    Params p[NG];
    int n;
    int tile_begin[NG + 1];
    // launch tiles from split_from on (a last, partial wave) are computed as
    // two 256 x 128 halves each, on two pairs (== tile_begin[n]: no split)
    int split_from;
};

template <int STAGES, int FMT, int NG>
__global__ void __launch_bounds__(kPairThreads, 1)
fp4_gemm_pair_kernel(const __grid_constant__ PairArgs<NG> args)
{
    constexpr bool MX = FMT == kMx;   // 32-element blocks (scale_vec::2X); else 16 (4X)
    using C = PairCfg<STAGES, MX>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BARS);
    // [0,S) full (leader), [S,2S) empty, [2S,3S) sf_full,
    // [3S] acc_full, [3S+1] acc_empty (leader), [3S+2] drain
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const uint32_t smem0 = smem_u32(smem);
    const uint32_t bar0 = smem_u32(bars);
    auto B_FULL = [&](int s) { return bar0 + 8u * s; };
    auto B_EMPTY = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto B_SFFULL = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
    const uint32_t acc_full = bar0 + 8u * (3 * STAGES);
    const uint32_t acc_empty = bar0 + 8u * (3 * STAGES + 1);
    const uint32_t drain = bar0 + 8u * (3 * STAGES + 2);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(B_FULL(s), C::FULL_ARRIVALS);
            mbar_init(B_EMPTY(s), 1);
            mbar_init(B_SFFULL(s), 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * kEpiWarps);
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();   // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    // work items: whole tiles below split_from, then two halves per tile
    const int tiles = args.split_from + 2 * (args.tile_begin[args.n] - args.split_from);
    // problem, M and N tile of work item t, and its column half: nh = 0 for a
    // whole 256 x 256 tile, 1 + h for the columns [128 h, 128 h + 128) of it
    auto locate = [&](int t, int& g, int& tm, int& tn, int& nh) {
        int ft = t;
        nh = 0;
        if (t >= args.split_from) {
            ft = args.split_from + ((t - args.split_from) >> 1);
            nh = 1 + ((t - args.split_from) & 1);
        }
        g = 0;
        if (NG > 1)
            while (g + 1 < args.n && ft >= args.tile_begin[g + 1]) ++g;
        const int lt = ft - args.tile_begin[g];
        // grouped raster: raster_gm consecutive M tiles sweep the N tiles
        // together (M fastest inside a group), so that the A row blocks of a
        // group stay in L2 while the B row blocks stream past them once per
        // group (raster_gm = tiles_m: plain M-fastest order)
        const int tiles_m = args.p[g].tiles_m;
        const int rg = args.p[g].raster_gm;
        const int span = rg * args.p[g].tiles_n;
        const int grp = lt / span, in = lt - grp * span;
        const int m0 = grp * rg;
        const int gm = min(tiles_m - m0, rg);
        tm = m0 + in % gm;
        tn = in / gm;
    };

    if (warp == 0) {
        // ---------------- producer (both CTAs, lane 0) ----------------
        if (lane == 0) {
            for (int g = 0; g < args.n; ++g) {
                asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&args.a[g])) : "memory");
                asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&args.b[g])) : "memory");
            }
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            pdl_wait();
            for (int t = pair; ok && t < tiles; t += npairs) {
                int g, tm, tn, nh;
                locate(t, g, tm, tn, nh);
                const Params& p = args.p[g];
                const int64_t sf_row_bytes = (int64_t)p.sf_col_tiles * SF_CHUNK;
                const int rta = tm * 2 + (int)rank;                // this CTA's 128-row A tile
                const bool has_sfa = rta < p.sfa_row_tiles;
                // B rows of the item: a half tile has the 128 from column
                // 128 h, each CTA's 64 the first rows of its 128-row box
                const int rtb0 = nh ? tn * 2 + nh - 1 : tn * 2;
                int nbh = 0;
                for (int h = 0; h < (nh ? 1 : 2); ++h)
                    if (rtb0 + h < p.sfb_row_tiles) ++nbh;
                const uint8_t* sfa_row = p.sfa + rta * sf_row_bytes;
                const uint8_t* sfb_row = p.sfb + (int64_t)rtb0 * sf_row_bytes;
                const int ya = rta * BM;
                const int yb = nh ? rtb0 * 128 + (int)rank * (PAIR_BHALF / 2) : tn * PAIR_BN + (int)rank * PAIR_BHALF;
                for (int ks = 0; ks < p.ks_total; ++ks) {
                    if (!wait_fast(B_EMPTY(stage), phase ^ 1u, abort_flag, ERR_EMPTY)) {
                        ok = false;
                        break;
                    }
                    const int nk = min(4, (p.K - ks * BK) / MMA_K);
                    const int nch = MX ? nk / 2 : nk;
                    const int ct0 = MX ? ks * 2 : ks * 4;
                    const uint32_t sf_bytes = (uint32_t)nch * SF_CHUNK;
                    const uint32_t st = smem0 + stage * C::STAGE_BYTES;
                    if (leader)
                        mbar_arrive_expect_tx(B_FULL(stage), 2u * (A_BYTES + C::B_BYTES));
                    const uint32_t full_leader = map_to_rank(B_FULL(stage), 0);
                    // the scale chunks first: they land before the operand tiles, so
                    // their staging into TMEM stays off the slot's critical path
                    mbar_arrive_expect_tx(B_SFFULL(stage), sf_bytes * ((has_sfa ? 1 : 0) + nbh));
                    if (has_sfa)
                        bulk_load(st + C::OFF_SFA, sfa_row + ct0 * SF_CHUNK, sf_bytes, B_SFFULL(stage));
                    if (nbh > 0)
                        bulk_load(st + C::OFF_SFB, sfb_row + ct0 * SF_CHUNK, sf_bytes, B_SFFULL(stage));
                    if (nbh > 1)
                        bulk_load(st + C::OFF_SFB + C::SFA_STAGE, sfb_row + sf_row_bytes + ct0 * SF_CHUNK,
                                  sf_bytes, B_SFFULL(stage));
                    tma_load_2d_pair(&args.a[g], full_leader, st, ks * BK_BYTES, ya);
                    tma_load_2d_pair(&args.b[g], full_leader, st + C::OFF_B, ks * BK_BYTES, yb);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            pdl_trigger();
            // On a give-up, give loads already issued time to land before the
            // CTAs meet at the final cluster barrier.
            if (!ok || *abort_flag) spin_ns(200000);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issue (leader CTA; lane 0 issues) ----------------
        // The issuing thread touches no mbarrier inside the loop: a probe or a
        // wait on a stage's barrier between two stages' MMAs leaves the
        // tensor pipe idle for 40-50 of the 512 cycles a 256-deep stage takes
        // (measured with the same loop on static operands).  The gatekeeper
        // warp does every wait and lets this warp through stage s by the
        // hardware named barrier 1 + s; tcgen05.fence::after_thread_sync then
        // orders the stage's MMAs after the operand tiles and scales the
        // gatekeeper's waits observed.  Each stage's slot is released by a
        // commit after its MMAs, the accumulator by a commit after the tile.
        if (leader) {
            const uint64_t adesc0 = desc_sw128(smem0);
            const uint64_t bdesc0 = desc_sw128(smem0 + C::OFF_B);
            constexpr uint32_t kDescPerStage = C::STAGE_BYTES >> 4;
            const uint32_t tsf0 = tmem_base + C::SF_COL0;
            int stage = 0;
            for (int t = pair; t < tiles; t += npairs) {
                int g, tm, tn, nh;
                locate(t, g, tm, tn, nh);
                const Params& p = args.p[g];
                const int kst = p.ks_total;
                const uint32_t n_mma = nh ? PAIR_BN / 2 : PAIR_BN;
                const uint32_t idesc0 = make_idesc_pair<FMT>(0, n_mma);
                const uint32_t idesc2 = make_idesc_pair<FMT>(2, n_mma);
                for (int ks = 0; ks < kst; ++ks) {
                    named_bar_sync(1 + stage, 64);
                    if (lane == 0) {
                        tc_fence_after();
                        const int nk = min(4, (p.K - ks * BK) / MMA_K);
                        const uint64_t ad = adesc0 + (uint64_t)(stage * kDescPerStage);
                        const uint64_t bd = bdesc0 + (uint64_t)(stage * kDescPerStage);
                        const uint32_t tsf = tsf0 + stage * C::SF_COLS;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            if (j < nk) {
                                const int chunk = MX ? (j >> 1) : j;
                                tc_mma_pair<MX>(tmem_base, ad + 2 * j, bd + 2 * j,
                                                (MX && (j & 1)) ? idesc2 : idesc0, tsf + 4 * chunk,
                                                tsf + C::SFA_COLS + chunk * 8, (j > 0 || ks > 0) ? 1u : 0u);
                            }
                        }
                        tc_commit_pair_both(B_EMPTY(stage));
                    }
                    __syncwarp();
                    if (++stage == STAGES) stage = 0;
                }
                if (lane == 0) tc_commit_pair_both(acc_full);
                __syncwarp();
            }
            if (lane == 0) {
                // every pair MMA issued here has completed before the TMEM is freed
                asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                 drain)
                             : "memory");
                wait_drain(drain, 0);
            }
        }
        __syncwarp();
    } else if (warp == kGateWarp) {
        // ---------------- gatekeeper (leader CTA, whole warp) ----------------
        // For each tile: the accumulator's release by both epilogues, then
        // per stage the full barrier (both CTAs' operand tiles and the 8
        // staging warps' scales); after each, the MMA warp is let through
        // the stage's named barrier.  A stage is refilled only after its MMAs
        // released it, so no named barrier has more than one arrival
        // pending.  After a failed (timed-out) wait the warp keeps arriving
        // without waiting, so that the MMA warp is never left blocked; the
        // timeout is recorded in the error word.
        if (leader) {
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int t = pair; t < tiles; t += npairs) {
                int g, tm, tn, nh;
                locate(t, g, tm, tn, nh);
                const int kst = args.p[g].ks_total;
                if (ok && !warp_wait(acc_empty, acc_phase ^ 1u, abort_flag, ERR_ACC_EMPTY)) ok = false;
                for (int ks = 0; ks < kst; ++ks) {
                    if (ok && !warp_wait(B_FULL(stage), phase, abort_flag, ERR_FULL)) ok = false;
                    named_bar_arrive(1 + stage, 64);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                acc_phase ^= 1u;
            }
        }
    } else if (warp < 6 || warp >= 10) {
        // ---------------- epilogue (warps 2..5 and 10..13, both CTAs) ----------------
        const int q = warp & 3;                      // TMEM lane quadrant
        const int half = warp >= 10 ? 1 : 0;         // accumulator columns [128 half, 128 half + 128)
        const int eb = half * 4 + q;                 // staging block
        pdl_wait();
        const uint32_t trow = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * 128);
        const uint32_t acc_empty_leader = map_to_rank(acc_empty, 0);
        uint32_t acc_phase = 0;
        for (int t = pair; t < tiles; t += npairs) {
            int g, tm, tn, nh;
            locate(t, g, tm, tn, nh);
            const Params& p = args.p[g];
            const float alpha = p.alpha ? *p.alpha : 1.0f;
            if (!warp_wait(acc_full, acc_phase, abort_flag, ERR_ACC_FULL)) break;
            tc_fence_after();
            if (nh && half) {
                // a half tile has 128 accumulator columns: the second-half
                // warps only hand the accumulator back
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (leader)
                        mbar_arrive(acc_empty);
                    else
                        mbar_arrive_cluster_relaxed(acc_empty_leader);
                }
                acc_phase ^= 1u;
                continue;
            }
            // four 32-column loads, two buffers: each load overlaps the
            // conversion of the previous chunk
            uint32_t packed[64];
            uint32_t ra[32], rb[32];
            auto convert = [&](const uint32_t (&r)[32], int c) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    packed[c * 16 + i] = pack_bf16x2(__fmul_rn(alpha, __uint_as_float(r[2 * i])),
                                                     __fmul_rn(alpha, __uint_as_float(r[2 * i + 1])));
            };
            tmem_ld32(trow, ra);
            tmem_wait_ld(ra);
            tmem_ld32(trow + 32, rb);
            convert(ra, 0);
            tmem_wait_ld(rb);
            tmem_ld32(trow + 64, ra);
            convert(rb, 1);
            tmem_wait_ld(ra);
            tmem_ld32(trow + 96, rb);
            convert(ra, 2);
            tmem_wait_ld(rb);
            // every column is in registers: hand the accumulator back before
            // converting the last chunk
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader)
                    mbar_arrive(acc_empty);
                else
                    mbar_arrive_cluster_relaxed(acc_empty_leader);
            }
            convert(rb, 3);
            // D through shared memory: the warp's 32 rows x 32 columns at a
            // time go to its staging block (64-byte rows; 16-byte chunk j of
            // row r at chunk j ^ ((r >> 1) & 3), the 64-byte swizzle), then
            // one lane stores the block with TMA, coalesced and clipped to D.
            const int y0 = (tm * 2 + (int)rank) * BM + q * 32;
            const int col0 = nh ? tn * PAIR_BN + (nh - 1) * 128 : tn * PAIR_BN + half * 128;
            const uint32_t blk = smem0 + C::OFF_EPI + eb * C::EPI_BLOCK;
            const uint32_t my_row = blk + lane * 64;
            const int sw = (lane >> 1) & 3;
            if (y0 < p.rows_a) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int x0 = col0 + c * 32;
                    if (x0 >= p.rows_b) break;
                    if (lane == 0) bulk_wait_read_all();   // the block's previous store has read it
                    __syncwarp();
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(my_row + ((j ^ sw) << 4)),
                                     "r"(packed[c * 16 + 4 * j]), "r"(packed[c * 16 + 4 * j + 1]),
                                     "r"(packed[c * 16 + 4 * j + 2]), "r"(packed[c * 16 + 4 * j + 3])
                                     : "memory");
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) tma_store_2d(&args.d[g], blk, x0, y0);
                }
            }
            acc_phase ^= 1u;
        }
        if (lane == 0) bulk_wait_all();   // every store of D has completed
        __syncwarp();
    } else {
        // ---------------- scale staging (warps 6..9, both CTAs) ----------------
        const uint32_t tq = tmem_base + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t full_leader0 = map_to_rank(B_FULL(0), 0);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = pair; ok && t < tiles; t += npairs) {
            int g, tm, tn, nh;
            locate(t, g, tm, tn, nh);
            const Params& p = args.p[g];
            const bool has_sfa = tm * 2 + (int)rank < p.sfa_row_tiles;
            // scale row tiles of B staged (a half tile has one)
            const int rtb0 = nh ? tn * 2 + nh - 1 : tn * 2;
            int nbh = 0;
            for (int h = 0; h < (nh ? 1 : 2); ++h)
                if (rtb0 + h < p.sfb_row_tiles) ++nbh;
            for (int ks = 0; ks < p.ks_total; ++ks) {
                if (!warp_wait(B_SFFULL(stage), phase, abort_flag, ERR_FULL)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nk = min(4, (p.K - ks * BK) / MMA_K);
                const int nch = MX ? nk / 2 : nk;
                const uint32_t st = smem0 + stage * C::STAGE_BYTES + lane * 16;
                const uint32_t tsf = tq + C::SF_COL0 + stage * C::SF_COLS;
                uint32_t a[4 * C::NCH];
#pragma unroll
                for (int j = 0; j < C::NCH; ++j) {
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (j < nch && has_sfa) v = ld_shared_v4(st + C::OFF_SFA + j * SF_CHUNK);
                    a[4 * j] = v.x;
                    a[4 * j + 1] = v.y;
                    a[4 * j + 2] = v.z;
                    a[4 * j + 3] = v.w;
                }
                uint32_t b[8 * C::NCH];
#pragma unroll
                for (int j = 0; j < C::NCH; ++j)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint4 v = make_uint4(0u, 0u, 0u, 0u);
                        if (j < nch && h < nbh)
                            v = ld_shared_v4(st + C::OFF_SFB + h * C::SFA_STAGE + j * SF_CHUNK);
                        b[(j * 2 + h) * 4] = v.x;
                        b[(j * 2 + h) * 4 + 1] = v.y;
                        b[(j * 2 + h) * 4 + 2] = v.z;
                        b[(j * 2 + h) * 4 + 3] = v.w;
                    }
                if constexpr (MX) {
                    tmem_st8(tsf, a);
                    tmem_st16(tsf + C::SFA_COLS, b);
                } else {
                    tmem_st16(tsf, a);
                    tmem_st32(tsf + C::SFA_COLS, b);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (leader)
                        mbar_arrive(B_FULL(stage));
                    else
                        mbar_arrive_cluster_relaxed(full_leader0 + 8u * stage);
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    }

    tc_fence_before();
    cluster_sync();   // all pair MMAs done, both epilogues finished reading TMEM
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(C::TMEM_COLS)
                     : "memory");
    }
}

// Self-test of the bounded wait used by every kernel above: one thread waits
// on a barrier that nothing will ever complete.  The wait gives up after
// kTimeoutNs, records the error word, and the kernel returns normally.
__global__ void bounded_wait_selftest_kernel()
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        wait_bounded(smem_u32(&bar), 0, reinterpret_cast<volatile int*>(&abort_flag), ERR_SELFTEST);
    }
}

// ------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }();
    return fn;
}

// 2-D map over a packed operand [rows x row_bytes] (uint8), box 128 bytes x
// box_rows, 128-byte swizzle, zero fill out of bounds.
// D [rows x cols] BF16 with leading dimension ld (elements), stored by the
// pair kernel's epilogue in 32 x 32 boxes with the 64-byte swizzle.
bool make_map_d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld)
{
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes, int box_rows)
{
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)BK_BYTES, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Raises the kernel's dynamic shared-memory limit once per device; the
// statics are distinct for every instantiation of the kernel template.
template <int BN, int STAGES, int FMT, bool STREAM_K>
cudaError_t set_smem_once(int bytes)
{
    static std::mutex mu;
    static uint64_t done_mask = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && ((done_mask >> dev) & 1ull)) return cudaSuccess;
    e = cudaFuncSetAttribute(fp4_gemm_kernel<BN, STAGES, FMT, STREAM_K>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev < 64) done_mask |= 1ull << dev;
    return e;
}

template <int BN, int STAGES, int FMT, bool STREAM_K>
cudaError_t launch_kernel(const CUtensorMap& ta, const CUtensorMap& tb, const Params& p, int grid,
                          cudaStream_t s)
{
    using C = Cfg<BN, STAGES>;
    cudaError_t e = set_smem_once<BN, STAGES, FMT, STREAM_K>(C::SMEM);
    if (e != cudaSuccess) {
        set_last_error("cudaFuncSetAttribute(max dynamic shared memory)", e);
        return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kThreadsFor<BN>, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, fp4_gemm_kernel<BN, STAGES, FMT, STREAM_K>, ta, tb, p);
    if (e != cudaSuccess) {
        cudaFuncAttributes fa{};
        cudaFuncGetAttributes(&fa, fp4_gemm_kernel<BN, STAGES, FMT, STREAM_K>);
        int dev = 0, optin = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cudaGetLastError();
        char buf[200];
        snprintf(buf, sizeof buf,
                 "GEMM kernel launch (grid %d, smem %d, optin %d, func max dyn %d, static %zu, regs %d)",
                 grid, C::SMEM, optin, fa.maxDynamicSharedSizeBytes, fa.sharedSizeBytes, fa.numRegs);
        set_last_error(buf, e);
    }
    return e;
}

constexpr int DECODE_BN = 16, DECODE_STAGES = 8;    // 22 KB per stage

int decode_max_seg(int units, int G, int ks_total)
{
    if (units == 0) return 1;
    const int span = (units + G - 1) / G;
    return (span - 1) / ks_total + 2;
}

// Decode schedule: G CTAs; the first sk_tiles weight tiles are split over all
// CTAs by K stage (stream-K), the remaining tiles (a multiple of G) run whole.
// sk_tiles is the remainder of tiles / G, plus G more when that remainder
// would give the CTAs fewer than two K stages each, so that no tile has a
// crowd of one-stage contributors.  Fewer tiles than CTAs: all stream-K.
struct DecodeSchedule {
    int G, sk_tiles, max_seg;
};

DecodeSchedule decode_schedule(int64_t tiles, int ks_total, int sm_count)
{
    DecodeSchedule d;
    const int64_t units = tiles * ks_total;
    d.G = (int)(units < sm_count ? units : sm_count);
    if (tiles <= d.G) {
        d.sk_tiles = (int)tiles;
    } else {
        int64_t sk = tiles % d.G;
        if (sk > 0 && sk * ks_total < 2 * (int64_t)d.G) sk += d.G;
        d.sk_tiles = (int)sk;
    }
    d.max_seg = decode_max_seg(d.sk_tiles * ks_total, d.G, ks_total);
    return d;
}

// Workspace of the decode kernel: a fixed 64 KB block of arrival counters,
// one per (weight tile, lane quadrant), at offset 0 for every shape, then the
// FP32 partials [CTA][segment][16][128].  The counters must be zero when a
// call starts and every completed call leaves them zero, so a workspace that
// was zeroed once serves any sequence of shapes: the partials of one shape
// never overlap the counters of another.
constexpr size_t kDecodeCounterBytes = 65536;
constexpr int64_t kDecodeMaxTiles = kDecodeCounterBytes / (4 * sizeof(int));   // N <= 524288

size_t decode_partials_bytes(int G, int max_seg)
{
    const size_t b = (size_t)G * max_seg * DECODE_BN * BM * sizeof(float);
    return (b + 255) / 256 * 256;
}

}  // namespace

int tensor_map_encoder_available() { return encoder() != nullptr; }

size_t decode_workspace_bytes(int64_t M, int64_t N, int64_t K, int sm_count)
{
    if (M > DECODE_BN || M <= 0 || N <= 0 || K <= 0 || sm_count <= 0) return 0;
    if ((N + BM - 1) / BM > kDecodeMaxTiles) return 0;
    const int ks_total = (int)((K + BK - 1) / BK);
    const DecodeSchedule d = decode_schedule((N + BM - 1) / BM, ks_total, sm_count);
    return kDecodeCounterBytes + decode_partials_bytes(d.G, d.max_seg);
}

static void fill_common(Params& p, const GemmArgs& a, int64_t rows_a, int64_t rows_b,
                        const uint8_t* sfa, const uint8_t* sfb)
{
    const int kb = block_size(a.fmt);
    p.sfa = sfa;
    p.sfb = sfb;
    p.rows_a = (int32_t)rows_a;
    p.rows_b = (int32_t)rows_b;
    p.K = (int32_t)a.K;
    p.ks_total = (int32_t)((a.K + BK - 1) / BK);
    p.sf_col_tiles = (int32_t)((a.K / kb + 3) / 4);
    p.sfa_row_tiles = (int32_t)((rows_a + 127) / 128);
    p.sfb_row_tiles = (int32_t)((rows_b + 127) / 128);
    p.alpha = a.alpha;
    p.D = a.D;
    p.ldd = a.ldd;
    p.ws = nullptr;
    p.counters = nullptr;
    p.act = nullptr;
    p.lda = 0;
    p.act_gs = nullptr;
    p.units = 0;
    p.sk_tiles = 0;
    p.a_static = 0;
    p.max_seg = 0;
    p.raster_gm = 1;
}

template <int STAGES, int FMT, int NG>
cudaError_t launch_pair_kernel(const PairArgs<NG>& args, int grid, cudaStream_t s)
{
    using C = PairCfg<STAGES, FMT == kMx>;
    auto kern = fp4_gemm_pair_kernel<STAGES, FMT, NG>;
    static std::mutex mu;
    static uint64_t done_mask = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!(dev < 64 && ((done_mask >> dev) & 1ull))) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
            if (e != cudaSuccess) {
                set_last_error("cudaFuncSetAttribute(pair kernel)", e);
                return e;
            }
            if (dev < 64) done_mask |= 1ull << dev;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kPairThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kern, args);
    if (e != cudaSuccess) set_last_error("pair GEMM kernel launch", e);
    return e;
}

constexpr int PAIR_STAGES_NV = 5;   // 38 KB per stage
constexpr int PAIR_STAGES_MX = 5;   // 35 KB per stage

// Fills problem slot g of a pair-kernel launch (tensor maps and Params).
template <int NG>
bool fill_pair_problem(PairArgs<NG>& args, int g, const GemmArgs& a)
{
    if (!make_map(&args.a[g], a.A, a.M, a.K / 2, BM) || !make_map(&args.b[g], a.B, a.N, a.K / 2, PAIR_BHALF) ||
        !make_map_d(&args.d[g], a.D, a.M, a.N, a.ldd))
        return false;
    Params& p = args.p[g];
    fill_common(p, a, a.M, a.N, a.sA, a.sB);
    p.tiles_m = (int32_t)((a.M + 255) / 256);
    p.tiles_n = (int32_t)((a.N + PAIR_BN - 1) / PAIR_BN);
    // tile order: plain M-fastest when all of A (codes and scales) fits in
    // about half of the L2 cache, else groups of M tiles whose A rows fit in
    // kRasterGroupBytes, so that B streams past each group once
    const int64_t a_tile_bytes = 256 * (a.K / 2 + a.K / block_size(a.fmt));
    int64_t rg = p.tiles_m;
    if (a_tile_bytes * p.tiles_m > (int64_t)(64 << 20))
        rg = (kRasterGroupBytes + a_tile_bytes / 2) / a_tile_bytes;
    p.raster_gm = (int32_t)(rg < 1 ? 1 : (rg > p.tiles_m ? p.tiles_m : rg));
    args.tile_begin[g + 1] = args.tile_begin[g] + p.tiles_m * p.tiles_n;
    return true;
}

template <int NG>
cudaError_t launch_pair(PairArgs<NG>& args, int fmt, const DeviceInfo& dev, cudaStream_t s)
{
    const int64_t tiles = args.tile_begin[args.n];
    if (tiles == 0) return cudaSuccess;
    const int64_t max_pairs = dev.sm_count / 2;
    // Tiles are dealt to the pairs round-robin, so a last wave of R < pairs
    // tiles leaves pairs idle for a whole tile.  When its halves fit on the
    // pairs (2R <= pairs) those R tiles are computed as 2R half tiles
    // (256 x 128), one per pair.  (A stage's fixed latency makes a half tile
    // take more than half a tile's time; the split still shortens the wave.)
    const int64_t rem = tiles % max_pairs;
    const bool split = NG == 1 && rem > 0 && 2 * rem <= max_pairs;
    args.split_from = (int)(split ? tiles - rem : tiles);
    const int64_t items = tiles + (split ? rem : 0);
    const int grid = 2 * (int)(items < max_pairs ? items : max_pairs);
    if (fmt == kMx) return launch_pair_kernel<PAIR_STAGES_MX, kMx, NG>(args, grid, s);
    if (fmt == kP1) return launch_pair_kernel<PAIR_STAGES_NV, kP1, NG>(args, grid, s);
    return launch_pair_kernel<PAIR_STAGES_NV, kNv, NG>(args, grid, s);
}

cudaError_t launch_gemm_prefill(const GemmArgs& a, const DeviceInfo& dev, cudaStream_t s)
{
    PairArgs<1> args;
    args.n = 1;
    args.tile_begin[0] = 0;
    if (!fill_pair_problem(args, 0, a)) {
        set_last_error("cuTensorMapEncodeTiled", cudaErrorInvalidValue);
        return cudaErrorInvalidValue;
    }
    return launch_pair(args, a.fmt, dev, s);
}

// Several problems per launch, kMaxGroups at a time; problems with M == 0 or
// N == 0 are skipped, K == 0 is handled by the caller.
cudaError_t launch_gemm_grouped(int n, const GemmArgs* a, const DeviceInfo& dev, cudaStream_t s)
{
    for (int i0 = 0; i0 < n; i0 += kMaxGroups) {
        PairArgs<kMaxGroups> args;
        args.n = 0;
        args.tile_begin[0] = 0;
        for (int i = i0; i < n && i < i0 + kMaxGroups; ++i) {
            if (a[i].M == 0 || a[i].N == 0 || a[i].K == 0) continue;
            if (!fill_pair_problem(args, args.n, a[i])) {
                set_last_error("cuTensorMapEncodeTiled", cudaErrorInvalidValue);
                return cudaErrorInvalidValue;
            }
            ++args.n;
        }
        if (args.n == 0) continue;
        const cudaError_t e = launch_pair(args, a[i0].fmt, dev, s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_gemm_decode(const GemmArgs& a, const DeviceInfo& dev, cudaStream_t s)
{
    // swap: the weight operand B [N x K] is the 128-row MMA side, the M <= 16
    // tokens form the N = 16 side
    CUtensorMap tw, tx;
    // (with the activation quantized in the kernel there is no packed
    // activation to map: the weights' map is passed in its place, unused)
    if (!make_map(&tw, a.B, a.N, a.K / 2, BM) ||
        !make_map(&tx, a.act ? a.B : a.A, a.act ? a.N : a.M, a.K / 2, DECODE_BN)) {
        set_last_error("cuTensorMapEncodeTiled", cudaErrorInvalidValue);
        return cudaErrorInvalidValue;
    }
    Params p;
    fill_common(p, a, a.N, a.M, a.sB, a.sA);
    p.tiles_m = (int32_t)((a.N + BM - 1) / BM);
    p.tiles_n = 1;
    const DecodeSchedule d = decode_schedule(p.tiles_m, p.ks_total, dev.sm_count);
    const int G = d.G;
    p.sk_tiles = d.sk_tiles;
    p.a_static = a.b_static ? 1 : 0;   // the weight operand B is the MMA A side here
    p.act = a.act;
    p.lda = a.lda;
    p.act_gs = a.act_gs;
    p.units = d.sk_tiles * p.ks_total;
    p.max_seg = d.max_seg;
    // the counters start at zero (caller's contract) and the kernel leaves
    // them at zero
    p.counters = static_cast<int*>(a.ws);
    p.ws = reinterpret_cast<float*>(static_cast<uint8_t*>(a.ws) + kDecodeCounterBytes);
    if (a.fmt == kMx)
        return launch_kernel<DECODE_BN, DECODE_STAGES, kMx, true>(tw, tx, p, G, s);
    if (a.fmt == kP1) return launch_kernel<DECODE_BN, DECODE_STAGES, kP1, true>(tw, tx, p, G, s);
    return launch_kernel<DECODE_BN, DECODE_STAGES, kNv, true>(tw, tx, p, G, s);
}

// ------------------------------------------------------------------------
// Allocation-free decode: the counters and split-K partials go to a fixed,
// file-scope device array instead of a caller-provided workspace.  Every
// device that loads the library holds these bytes until the process exits.
// The array is zero at load, which is the state the counters need, and each
// completed call leaves them zero; two such calls that overlap on the GPU
// (different streams) race on it.
// ------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Device address of g_decode_scratch in the current context.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device with that device current and cached together with the
// context it belongs to; a new context on the device (e.g. after
// cudaDeviceReset) makes the lookup run again.
cudaError_t noalloc_scratch(void** out)
{
    static std::mutex mu;
    static void* cache[64] = {};
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
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess) return e;
    if (dev < 64) {
        cache[dev] = ptr;
        cache_ctx[dev] = ctx;
    }
    *out = ptr;
    return cudaSuccess;
}

cudaError_t clear_noalloc_counters(cudaStream_t s)
{
    void* ptr = nullptr;
    cudaError_t e = noalloc_scratch(&ptr);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(ptr, 0, kDecodeCounterBytes, s);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(s);
}

cudaError_t launch_wait_selftest(cudaStream_t s)
{
    bounded_wait_selftest_kernel<<<1, 32, 0, s>>>();
    return cudaGetLastError();
}

cudaError_t read_and_clear_error_word(unsigned int* word)
{
    cudaError_t e = cudaMemcpyFromSymbol(word, g_fp4_error_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    if (*word) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_fp4_error_word, &zero, sizeof(unsigned int));
    }
    return e;
}

}  // namespace fp4
