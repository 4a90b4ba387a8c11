// scaled_mm.cu -- fp8 x fp8 matrix products on the sm_100a tensor cores.
//
// Two products of the same shape, D[M][N] = A[M][K] * B[N][K]^T, both
// operands fp8 codes (A: activations, B: a weight as it is stored, [out
// features][in features]), each stored K-contiguous or, for the per-tensor
// product, MN-contiguous ([K][M] / [K][N] row-major: the transposed operands
// of linear_fp8's backward, read where they lie):
//   per-tensor scales (ColossalAI colossalai/quantization/fp8.py,
//     _LinearFp8.forward: torch._scaled_mm with the scale_inv of each operand)
//       D[m][n] = T(fl(acc[m][n] * fl(sa * sb)) + bias[n])
//   fine-grained scales (DeepEP per_token_cast_to_fp8 activations, one
//     scale_inv per 1 x 128 group: sa[M][ceil(K/128)]; a DeepSeek-V3 weight
//     with one scale_inv per 128 x 128 block: sb[ceil(N/128)][ceil(K/128)])
//       D[m][n] = T(sum over k-blocks kb of fl(sa[m][kb] * sb[n/128][kb]) *
//                   acc_kb[m][n]  + bias[n])
// where acc is the fp32 tensor-core sum of the fp8 products.
//
// Design (one persistent CTA per SM, warp-specialised):
//   warp 0      TMA producer: 128 x 128-byte tiles of A and BN x 128-byte
//               tiles of B (128-byte swizzle) into a shared-memory ring
//   warp 1      allocates 512 TMEM columns; one lane issues
//               tcgen05.mma.kind::f8f6f4 (M 128, N BN, K 32) into one of the
//               128 x BN fp32 TMEM accumulators and commits each stage back
//               to the producer and each finished accumulator to the epilogue
//   warps 2-9   epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32 * (w % 4) .. + 31, column group (w - 2) / 4), every
//               lane polling the accumulator's barrier; scaling, bias,
//               conversion, 32-byte stores (TMEM loads double-buffered in
//               32-column chunks).  With fine-grained scales the MMA warp
//               commits every 128-deep k-block into a fresh accumulator and
//               the epilogue folds it into registers with that block's scale
//               (packed fp32x2 FMAs, TMEM loads double-buffered in 16-column
//               chunks; warps whose rows all lie past M only take part in the
//               handshake), while the tensor cores fill the other
//               accumulator.
// Tiles are 128 x BN of D, visited in bands of 32 row-tiles so that the CTAs
// working at one time share A and B tiles in L2.  Per-tensor products with
// enough rows take 256 x 256 tiles on CTA pairs instead (namespace pair below:
// one tcgen05.mma.cta_group::2 per k step across two SMs) when those tiles
// give two CTAs each to nine tenths of the SMs.  A one-CTA 256 x 256 variant
// (two M 128 MMAs per k step share the B tile; see Shape) serves builds
// without pairs (FP8Q_PAIRS=0).  A product of fewer than 128 rows loads only
// its rows of A (rounded up to 16).
//
// Every wait on an mbarrier is bounded (a few seconds of global time).  A
// wait that runs out sets a flag in shared memory that ends the other roles'
// waits too, ORs a code into the caller's status word, drains the copies and
// tensor-core operations this CTA has in flight, frees its TMEM and returns.
#include <cuda.h>

#include <cstring>

#include "fp8q_device.cuh"
#include "fp8q_internal.h"

namespace fp8q {
namespace mm {

constexpr int BM = 128;         // rows of A (and of D) per tile
constexpr int BK = 128;         // k per stage: one 128-byte swizzle row, one scale block
constexpr int kTmemCols = 512;  // all of TMEM, split into kAccBufs accumulators
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kGroupM = 32;     // row-tiles per raster band

// Tile shapes.  BN = 256: 128 x 256 tiles, two TMEM accumulators (with
// per-tensor scales one tile's epilogue overlaps the next tile's k-loop; with
// fine-grained scales one k-block's fold overlaps the next block's MMAs), a
// 4-stage ring: the shape for products with enough tiles to fill the GPU.
// BN = 128: 128 x 128 tiles, four accumulators, a 6-stage ring, for products
// of at most 128 rows (decode-sized activations), where 256-wide tiles would
// leave SMs without a share of the weight to stream.  Measured on B200 for
// large products: 128 x 128 tiles lose a quarter of the fine-grained
// throughput, since the narrower MMA reads twice the operand bytes per flop.
// MT = 256 (per-tensor scales only): 256 x 256 tiles, two M 128 MMAs per k
// step sharing the B tile, the two 128 x 256 accumulators filling TMEM (one
// buffer: each tile's epilogue is not overlapped), a 3-stage ring -- a third
// fewer operand bytes per flop than 128 x 256 tiles.
template <int BN_, int MT_ = 128> struct Shape {
    static constexpr int BN = BN_;                          // rows of B (columns of D) per tile
    static constexpr int MT = MT_;                          // rows of A (and of D) per tile
    static constexpr int kATile = MT_ * BK;
    static constexpr int kStages = MT_ == 256 ? 3 : (BN_ == 256 ? 4 : 6);
    static constexpr int kAccBufs = MT_ == 256 ? 1 : kTmemCols / BN;
    static constexpr int kColsPerWarp = BN / (kEpiWarps / 4);   // tile columns one epilogue warp owns
    static constexpr int kBBytes = BN * BK;
    static constexpr int kStageBytes = kATile + kBBytes;
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /* alignment slack */ + 256 /* barriers */;
};
constexpr uint64_t kWaitLimitNs = 4000000000ull;   // every wait's default limit
#ifndef FP8Q_PAIRS
#define FP8Q_PAIRS 1
#endif

// status bits ORed into the caller's status word when a wait runs out
enum : uint32_t { kTimeoutProducer = 1u, kTimeoutMma = 2u, kTimeoutEpilogue = 4u, kTimeoutDrain = 8u };
static_assert(kTimeoutProducer == FP8Q_WAIT_PRODUCER && kTimeoutMma == FP8Q_WAIT_MMA &&
              kTimeoutEpilogue == FP8Q_WAIT_EPILOGUE && kTimeoutDrain == FP8Q_WAIT_DRAIN, "status bits");

struct Params {
    int M, N, K;
    int num_kb;                 // ceil(K / BK)
    int tiles_m, tiles_n;
    const float* sa;            // per-tensor: [1]; fine-grained: [M][sa_ld]
    const float* sb;            // per-tensor: [1]; fine-grained: [ceil(N/128)][sb_ld]
    int sa_ld, sb_ld;
    const void* bias;           // [N] of the output type, or null
    void* d;                    // [M][N]
    int vec_store;              // D rows 32-byte aligned (base and row pitch)
    int stage_tx;               // bytes one stage's TMA boxes bring
    int a_mn, b_mn;             // operand stored MN-major ([K][M] / [K][N] row-major), else K-major
    uint32_t* status;           // optional status word
    uint64_t wait_limit_ns;     // bound of every wait (kWaitLimitNs unless a test sets it)
    int stall_kb;               // test hook: k-block of each CTA's first tile whose copies are left out (-1: none)
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}
// One try: the thread may be suspended in hardware until the phase completes
// or kTrySuspendNs pass, rather than spinning -- the polling warps then take
// no issue slots or shared-memory bandwidth from the rest of the SM while
// they wait (measured on B200: the fine-grained product 1.5% faster).
constexpr uint32_t kTrySuspendNs = 100000;
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity), "r"(kTrySuspendNs) : "memory");
    return ok != 0;
}
// Wait for the phase of `bar` with the given parity; false if the wait ran
// out of time or another role of this CTA has already given up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (global_ns() - t0 > limit_ns) return false;
    }
}
// the same wait, ignoring the abort flag (used to drain work in flight)
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];"
                 :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major operand tile written by TMA
// with the 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes
// apart (stride byte offset), leading byte offset unused (encoded 1), the
// Blackwell descriptor version 1, layout 2 = 128-byte swizzle.  The tile
// base is 1024-byte aligned; a k offset inside the 128-byte row moves the
// start address only.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    return static_cast<uint64_t>((addr >> 4) & 0x3FFFu)
         | (static_cast<uint64_t>(1) << 16)
         | (static_cast<uint64_t>(1024 >> 4) << 32)
         | (static_cast<uint64_t>(1) << 46)
         | (static_cast<uint64_t>(2) << 61);
}
// The same for an MN-major operand tile: each 128-byte row holds 128 M (or N)
// elements of one k, TMA writes 128 x 128-byte boxes (one per 128 M or N),
// 8-row k groups are 1024 bytes apart (stride byte offset) and successive
// 128-wide M or N boxes 16384 bytes apart (leading byte offset).  A k step of
// 32 moves the start address by 32 rows, 4096 bytes.
constexpr int kMnAtomBytes = 128 * BK;
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t addr) {
    return static_cast<uint64_t>((addr >> 4) & 0x3FFFu)
         | (static_cast<uint64_t>(kMnAtomBytes >> 4) << 16)
         | (static_cast<uint64_t>(1024 >> 4) << 32)
         | (static_cast<uint64_t>(1) << 46)
         | (static_cast<uint64_t>(2) << 61);
}
// Instruction descriptor of kind::f8f6f4: D fp32 (bits 4-5 = 1), A and B
// formats (bits 7-9, 10-12: 0 e4m3, 1 e5m2), A and B MN-major (bits 15, 16;
// 0 = K-major), N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t instr_desc(int fa, int fb, int bn, int a_mn = 0, int b_mn = 0) {
    return (1u << 4) | (static_cast<uint32_t>(fa) << 7) | (static_cast<uint32_t>(fb) << 10)
         | (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(b_mn) << 16)
         | (static_cast<uint32_t>(bn >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);
}
__device__ __forceinline__ void mma_f8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// arrive on `bar` once every tcgen05 operation this thread issued so far has completed
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(bar) : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns of TMEM into 32 registers per thread
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32"
                 " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
                   "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
                   "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
    // the registers pass through the wait, so no use of them can be scheduled before it
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
                   "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
                   "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 16 consecutive columns, issued without waiting: tmem_wait16 on
// the same registers completes it (and every other load still in flight)
__device__ __forceinline__ void tmem_ld16_async(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32"
                 " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15])
                 :: "memory");
}

// 32 lanes x 32 consecutive columns, issued without waiting (completed by
// tmem_wait32 on the same registers)
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32"
                 " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
                   "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
                   "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait32(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
                   "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
                   "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :: "memory");
}

// ---------------------------------------------------------------------------
// epilogue stores: 32 consecutive columns of one row of D
// ---------------------------------------------------------------------------
template <int YT> struct OutT;
template <> struct OutT<kF32> { using T = float; };
template <> struct OutT<kF16> { using T = __half; };
template <> struct OutT<kBF16> { using T = __nv_bfloat16; };

template <int YT> __device__ __forceinline__ float load_bias(const void* bias, int n) {
    if constexpr (YT == kF32) return __ldg(static_cast<const float*>(bias) + n);
    else if constexpr (YT == kF16) return __half2float(__ldg(static_cast<const __half*>(bias) + n));
    else return __bfloat162float(__ldg(static_cast<const __nv_bfloat16*>(bias) + n));
}

template <int YT> __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if constexpr (YT == kF16) {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    } else {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
}

template <int YT>
__device__ __forceinline__ void store_chunk(const Params& p, int row, int col0, const float (&v)[32]) {
    using T = typename OutT<YT>::T;
    T* drow = static_cast<T*>(p.d) + static_cast<int64_t>(row) * p.N;
    if (p.vec_store && col0 + 32 <= p.N) {
        if constexpr (YT == kF32) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(v[c * 8 + i]);
                st_v8(drow + col0 + c * 8, w);
            }
        } else {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) w[i] = pack2<YT>(v[c * 16 + 2 * i], v[c * 16 + 2 * i + 1]);
                st_v8(drow + col0 + c * 16, w);
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (col0 + i < p.N) {
                if constexpr (YT == kF32) drow[col0 + i] = v[i];
                else if constexpr (YT == kF16) drow[col0 + i] = __float2half_rn(v[i]);
                else drow[col0 + i] = __float2bfloat16_rn(v[i]);
            }
        }
    }
}

__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int& mb, int& nb) {
    const int band = t / (kGroupM * tiles_n);
    const int first = band * kGroupM;
    const int gm = min(tiles_m - first, kGroupM);
    const int local = t - band * kGroupM * tiles_n;
    mb = first + local % gm;
    nb = local / gm;
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int YT, bool FINE, int BN_, int MT_>
__global__ void __launch_bounds__(kThreads, 1)
scaled_mm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 const Params p, const uint32_t idesc) {
    constexpr int BN = Shape<BN_, MT_>::BN;
    constexpr int kStages = Shape<BN_, MT_>::kStages;
    constexpr int kAccBufs = Shape<BN_, MT_>::kAccBufs;
    constexpr int kColsPerWarp = Shape<BN_, MT_>::kColsPerWarp;
    constexpr int kBBytes = Shape<BN_, MT_>::kBBytes;
    constexpr int kATile = Shape<BN_, MT_>::kATile;
    constexpr int kSub = MT_ / BM;                 // M 128 sub-tiles (MMAs per k step, accumulators per tile)
    static_assert(!FINE || MT_ == BM, "fine-grained scales use 128-row tiles");
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_abort;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * kATile;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kStages * kBBytes);
    // bars: full[kStages], empty[kStages], tfull[kAccBufs], tempty[kAccBufs], drain
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 2 * kAccBufs + 1);
    const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * kStages;
    const uint32_t tfull0 = empty0 + 8 * kStages, tempty0 = tfull0 + 8 * kAccBufs;
    const uint32_t drain_bar = tempty0 + 8 * kAccBufs;
    volatile int* abort = &s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(tfull0 + 8 * b, 1);
            mbar_init(tempty0 + 8 * b, kEpiWarps);
        }
        mbar_init(drain_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        prefetch_tensormap(&map_a);
        prefetch_tensormap(&map_b);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    pdl_begin();

    const int tiles = p.tiles_m * p.tiles_n;
    uint32_t fail = 0;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int64_t issued = 0;
            for (int t = blockIdx.x; t < tiles && !fail; t += gridDim.x) {
                int mb, nb;
                tile_coords(t, p.tiles_m, p.tiles_n, mb, nb);
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort, p.wait_limit_ns)) { fail = kTimeoutProducer; break; }
                    const uint32_t fb = full0 + 8 * stage;
                    mbar_arrive_expect_tx(fb, static_cast<uint32_t>(p.stage_tx));
                    if (kb == p.stall_kb && t == static_cast<int>(blockIdx.x)) {
                        // test hook: this stage's bytes never arrive, so every
                        // wait that depends on them runs out
                        ++issued;
                        if (++stage == kStages) { stage = 0; phase ^= 1u; }
                        continue;
                    }
                    if (p.a_mn) {
#pragma unroll
                        for (int sub = 0; sub < kSub; ++sub)
                            tma_load_2d(smem_u32(sA + stage * kATile + sub * kMnAtomBytes), &map_a,
                                        mb * MT_ + sub * BM, kb * BK, fb);
                    } else {
                        tma_load_2d(smem_u32(sA + stage * kATile), &map_a, kb * BK, mb * MT_, fb);
                    }
                    if (p.b_mn) {
#pragma unroll
                        for (int h = 0; h < BN / 128; ++h)
                            tma_load_2d(smem_u32(sB + stage * kBBytes + h * kMnAtomBytes), &map_b, nb * BN + 128 * h,
                                        kb * BK, fb);
                    } else {
                        tma_load_2d(smem_u32(sB + stage * kBBytes), &map_b, kb * BK, nb * BN, fb);
                    }
                    ++issued;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (fail) *abort = 1;
            // every copy this thread issued has landed before the CTA exits
            for (int s = 0; s < kStages; ++s) {
                const bool used = s < stage || issued >= kStages;
                if (used && !mbar_wait_drain(full0 + 8 * s, s < stage ? phase : phase ^ 1u, p.wait_limit_ns)) fail |= kTimeoutDrain;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int t = blockIdx.x; t < tiles && !fail; t += gridDim.x) {
                if (p.num_kb == 0) continue;
                if (!FINE) {
                    if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort, p.wait_limit_ns)) { fail = kTimeoutMma; break; }
                    tc_fence_after();
                }
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (FINE) {
                        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort, p.wait_limit_ns)) { fail = kTimeoutMma; break; }
                        tc_fence_after();
                    }
                    if (!mbar_wait(full0 + 8 * stage, phase, abort, p.wait_limit_ns)) { fail = kTimeoutMma; break; }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * kATile), b0 = smem_u32(sB + stage * kBBytes);
#pragma unroll
                    for (int j = 0; j < BK / 32; ++j) {
                        const uint32_t accumulate = FINE ? (j > 0) : (kb > 0 || j > 0);
                        const uint64_t bd = p.b_mn ? smem_desc_mn_sw128(b0 + 4096 * j) : smem_desc_sw128(b0 + 32 * j);
#pragma unroll
                        for (int sub = 0; sub < kSub; ++sub) {
                            // sub-tile sub: rows 128 sub .. of A, its own accumulator
                            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>((acc + sub) * BN);
                            const uint64_t ad = p.a_mn ? smem_desc_mn_sw128(a0 + sub * kMnAtomBytes + 4096 * j)
                                                       : smem_desc_sw128(a0 + sub * BM * BK + 32 * j);
                            mma_f8f6f4(d_tmem, ad, bd, idesc, accumulate);
                        }
                    }
                    mma_commit(empty0 + 8 * stage);
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                    if (FINE) {
                        mma_commit(tfull0 + 8 * acc);
                        if (++acc == kAccBufs) { acc = 0; acc_phase ^= 1u; }
                    }
                }
                if (fail) break;
                if (!FINE) {
                    mma_commit(tfull0 + 8 * acc);
                    if (++acc == kAccBufs) { acc = 0; acc_phase ^= 1u; }
                }
            }
            if (fail) *abort = 1;
            // every tensor-core operation this thread issued has completed
            mma_commit(drain_bar);
            if (!mbar_wait_drain(drain_bar, 0, p.wait_limit_ns)) fail |= kTimeoutDrain;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 2;
        const int quarter = warp & 3;                 // TMEM lanes this warp may read
        const int cgrp = ew >> 2;                     // which kColsPerWarp-wide group of the tile's columns
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        int acc = 0;
        uint32_t acc_phase = 0;
        float scale = 0.0f;
        if (!FINE) scale = __fmul_rn(__ldg(p.sa), __ldg(p.sb));
        for (int t = blockIdx.x; t < tiles && !fail; t += gridDim.x) {
            int mb, nb;
            tile_coords(t, p.tiles_m, p.tiles_n, mb, nb);
            const int row = mb * MT_ + quarter * 32 + lane;
            const int col_base = nb * BN + cgrp * kColsPerWarp;
            if (!FINE) {
                if (p.num_kb > 0) {
                    const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(tfull0 + 8 * acc, acc_phase, abort, p.wait_limit_ns));
                    if (!ok) { fail = kTimeoutEpilogue; break; }
                    tc_fence_after();
                }
                // kSub x kColsPerWarp / 32 chunks of 32 columns, double-buffered:
                // the load of chunk j + 1 is in flight while chunk j is scaled
                // and stored
                constexpr int kChunks = kSub * (kColsPerWarp / 32);
                const uint32_t col_addr = tmem_base + lane_addr + static_cast<uint32_t>(acc * BN + cgrp * kColsPerWarp);
                uint32_t r0[32], r1[32];
                if (p.num_kb > 0) {
                    tmem_ld32_async(col_addr, r0);
                    tmem_wait32(r0);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) r0[i] = r1[i] = 0u;
                }
#pragma unroll
                for (int j = 0; j < kChunks; ++j) {
                    const int sub = j / (kColsPerWarp / 32), c = j % (kColsPerWarp / 32);
                    uint32_t (&cur)[32] = (j & 1) ? r1 : r0;
                    uint32_t (&nxt)[32] = (j & 1) ? r0 : r1;
                    if (p.num_kb > 0 && j + 1 < kChunks) {
                        const int sub1 = (j + 1) / (kColsPerWarp / 32), c1 = (j + 1) % (kColsPerWarp / 32);
                        tmem_ld32_async(col_addr + static_cast<uint32_t>(sub1 * BN + c1 * 32), nxt);
                    }
                    const int srow = row + sub * BM;
                    const int col0 = col_base + c * 32;
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(__uint_as_float(cur[i]), scale);
                    if (p.bias) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (col0 + i < p.N) v[i] = __fadd_rn(v[i], load_bias<YT>(p.bias, col0 + i));
                    }
                    if (srow < p.M && col0 < p.N) store_chunk<YT>(p, srow, col0, v);
                    if (p.num_kb > 0 && j + 1 < kChunks) tmem_wait32(nxt);
                }
                if (p.num_kb > 0) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
                    if (++acc == kAccBufs) { acc = 0; acc_phase ^= 1u; }
                }
            } else {
                // this warp's kColsPerWarp columns of its 32 rows, as fp32 pairs
                float2 accum[kColsPerWarp / 2];
#pragma unroll
                for (int i = 0; i < kColsPerWarp / 2; ++i) accum[i] = make_float2(0.0f, 0.0f);
                const bool row_ok = row < p.M;
                const bool warp_rows_live = row - lane < p.M;    // the warp's first row
                const bool blk_ok = col_base < p.N;
                const float* sa_row = p.sa + static_cast<int64_t>(row_ok ? row : 0) * p.sa_ld;
                const float* sb_row = p.sb + static_cast<int64_t>(blk_ok ? col_base / 128 : 0) * p.sb_ld;
                float sa_next = (row_ok && p.num_kb > 0) ? __ldg(sa_row) : 0.0f;
                float sb_next = (blk_ok && p.num_kb > 0) ? __ldg(sb_row) : 0.0f;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    const float s = __fmul_rn(sa_next, sb_next);
                    if (kb + 1 < p.num_kb) {
                        sa_next = row_ok ? __ldg(sa_row + kb + 1) : 0.0f;
                        sb_next = blk_ok ? __ldg(sb_row + kb + 1) : 0.0f;
                    }
                    // every lane polls; the vote keeps the warp converged
                    const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(tfull0 + 8 * acc, acc_phase, abort, p.wait_limit_ns));
                    if (!ok) { fail = kTimeoutEpilogue; break; }
                    tc_fence_after();
                    if (!warp_rows_live) {
                        // every row of this warp is past M (decode-sized
                        // products): nothing to fold, only the handshake
                        __syncwarp();
                        if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
                        if (++acc == kAccBufs) { acc = 0; acc_phase ^= 1u; }
                        continue;
                    }
                    // 8 chunks of 16 columns, double-buffered: the load of chunk
                    // c + 1 is in flight while chunk c is folded in with packed
                    // fused multiply-adds (each lane the same as __fmaf_rn)
                    const uint32_t col_addr = tmem_base + lane_addr + static_cast<uint32_t>(acc * BN + cgrp * kColsPerWarp);
                    const float2 s2 = make_float2(s, s);
                    uint32_t r0[16], r1[16];
                    tmem_ld16_async(col_addr, r0);
                    tmem_wait16(r0);
#pragma unroll
                    for (int c = 0; c < kColsPerWarp / 16; ++c) {
                        uint32_t (&cur)[16] = (c & 1) ? r1 : r0;
                        uint32_t (&nxt)[16] = (c & 1) ? r0 : r1;
                        if (c + 1 < kColsPerWarp / 16) tmem_ld16_async(col_addr + 16 * (c + 1), nxt);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            accum[c * 8 + i] = __ffma2_rn(make_float2(__uint_as_float(cur[2 * i]),
                                                                      __uint_as_float(cur[2 * i + 1])),
                                                          s2, accum[c * 8 + i]);
                        if (c + 1 < kColsPerWarp / 16) tmem_wait16(nxt);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
                    if (++acc == kAccBufs) { acc = 0; acc_phase ^= 1u; }
                }
                if (fail) break;
#pragma unroll
                for (int c = 0; c < kColsPerWarp / 32; ++c) {
                    float v[32];
                    const int col0 = col_base + c * 32;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        v[2 * i] = accum[c * 16 + i].x;
                        v[2 * i + 1] = accum[c * 16 + i].y;
                    }
                    if (p.bias) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (col0 + i < p.N) v[i] = __fadd_rn(v[i], load_bias<YT>(p.bias, col0 + i));
                    }
                    if (row_ok && col0 < p.N) store_chunk<YT>(p, row, col0, v);
                }
            }
        }
        if (fail && lane == 0) *abort = 1;
    }

    if (fail && p.status && lane == 0) atomicOr(p.status, fail);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// CTA pairs (per-tensor scales, either operand K- or MN-major): the two CTAs of a
// cluster compute one 256 x 256 tile with tcgen05.mma.cta_group::2 (M 256,
// N 256, K 32).  Each CTA loads its own 128 rows of A and its own 128 rows of
// B (half of the tile's N) into its shared memory, so a CTA reads a quarter
// fewer operand bytes per flop than a 128 x 256 tile on one SM; each CTA's
// TMEM holds its 128 rows x 256 columns of the tile, two buffers of it, so one
// tile's epilogue overlaps the next tile's k-loop.  The even CTA of the pair
// (the leader) expects both CTAs' bytes on its stage barriers and issues the
// MMAs; its commits release the stages and hand over finished accumulators
// in both CTAs at once (commit with .multicast::cluster); both CTAs' epilogue
// warps hand their accumulator back on the leader's barrier.  No load uses
// multicast: every CTA fetches its own tiles.
// ---------------------------------------------------------------------------
namespace pair {

constexpr int kStages = 6;
constexpr int BN = 256;                         // columns of D per tile (B rows, both CTAs together)
constexpr int kHalfB = BN / 2;                  // B rows one CTA loads
constexpr int kATile = BM * BK;                 // 16 KB: this CTA's 128 rows of A
constexpr int kBTile = kHalfB * BK;             // 16 KB: this CTA's half of B
constexpr int kAccBufs = 2;
constexpr int kTmemCols = 512;
constexpr int kColsPerWarp = BN / (kEpiWarps / 4);
constexpr int kSmemBytes = kStages * (kATile + kBTile) + 1024 + 256;
// clears the CTA-rank bit of a shared::cluster address: the same offset in the even CTA
constexpr uint32_t kLeaderMask = 0xFEFFFFFFu;

__device__ __forceinline__ uint32_t cta_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// a 2-D box into this CTA's shared memory, its bytes counted on the leader's barrier
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile("cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];"
                 :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar & kLeaderMask)
                 : "memory");
}
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// arrive on `bar` in both CTAs of the pair once this thread's MMAs so far have completed
__device__ __forceinline__ void commit_both(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 :: "r"(bar), "h"(static_cast<uint16_t>(3)) : "memory");
}
__device__ __forceinline__ void commit_local(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" :: "r"(bar) : "memory");
}
// arrive on the leader's barrier at the offset of `bar`
__device__ __forceinline__ void arrive_leader(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" :: "r"(bar & kLeaderMask) : "memory");
}

template <int YT>
__global__ void __launch_bounds__(kThreads, 1)
scaled_mm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const Params p, const uint32_t idesc) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_abort;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * kATile;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kStages * kBTile);
    // bars: full[kStages], empty[kStages], tfull[kAccBufs], tempty[kAccBufs], drain
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 2 * kAccBufs + 1);
    const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * kStages;
    const uint32_t tfull0 = empty0 + 8 * kStages, tempty0 = tfull0 + 8 * kAccBufs;
    const uint32_t drain_bar = tempty0 + 8 * kAccBufs;
    volatile int* abort = &s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cta_rank();
    const bool leader = rank == 0;
    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full0 + 8 * s, 1);           // the leader's expect-tx arrival, bytes of both CTAs
            mbar_init(empty0 + 8 * s, 1);          // the leader's commit
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(tfull0 + 8 * b, 1);          // the leader's commit
            mbar_init(tempty0 + 8 * b, 2 * kEpiWarps);   // every epilogue warp of both CTAs (leader's copy)
        }
        mbar_init(drain_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        prefetch_tensormap(&map_a);
        prefetch_tensormap(&map_b);
    }
    // the peer's barriers exist before anything signals them
    cluster_sync();
    if (warp == 1) {
        // both CTAs allocate, from the same warp, into the same slot offset
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    pdl_begin();

    const int tiles = p.tiles_m * p.tiles_n;          // 256 x 256 tiles
    const int pair_id = blockIdx.x >> 1, pairs = gridDim.x >> 1;
    uint32_t fail = 0;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int64_t issued = 0;
            for (int t = pair_id; t < tiles && !fail; t += pairs) {
                int mb, nb;
                tile_coords(t, p.tiles_m, p.tiles_n, mb, nb);
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort, p.wait_limit_ns)) { fail = kTimeoutProducer; break; }
                    const uint32_t fb = full0 + 8 * stage;
                    if (leader) mbar_arrive_expect_tx(fb, static_cast<uint32_t>(2 * (kATile + kBTile)));
                    if (leader && kb == p.stall_kb && t == pair_id) {
                        // test hook: the leader's half of this stage never arrives, so the
                        // stage never completes and every wait that depends on it runs out
                        ++issued;
                        if (++stage == kStages) { stage = 0; phase ^= 1u; }
                        continue;
                    }
                    // K-major: boxes of 128 rows x 128 k; MN-major: 128 k x 128 rows
                    const int m0 = mb * 2 * BM + static_cast<int>(rank) * BM;
                    const int n0 = nb * BN + static_cast<int>(rank) * kHalfB;
                    if (p.a_mn) tma_load_2d_pair(smem_u32(sA + stage * kATile), &map_a, m0, kb * BK, fb);
                    else tma_load_2d_pair(smem_u32(sA + stage * kATile), &map_a, kb * BK, m0, fb);
                    if (p.b_mn) tma_load_2d_pair(smem_u32(sB + stage * kBTile), &map_b, n0, kb * BK, fb);
                    else tma_load_2d_pair(smem_u32(sB + stage * kBTile), &map_b, kb * BK, n0, fb);
                    ++issued;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (fail) *abort = 1;
            // every stage this CTA filled has been consumed by the pair's MMAs
            // (so its copies have landed) before the CTA moves on
            for (int s = 0; s < kStages; ++s) {
                const bool used = s < stage || issued >= kStages;
                // (a stage refilled in this lap waits for the release of that fill, parity
                // `phase`; one last filled in the previous lap, parity `phase ^ 1`)
                if (used && !mbar_wait_drain(empty0 + 8 * s, s < stage ? phase : phase ^ 1u, p.wait_limit_ns))
                    fail |= kTimeoutDrain;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int t = pair_id; t < tiles && !fail; t += pairs) {
                if (p.num_kb == 0) continue;
                if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort, p.wait_limit_ns)) { fail = kTimeoutMma; break; }
                tc_fence_after();
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!mbar_wait(full0 + 8 * stage, phase, abort, p.wait_limit_ns)) { fail = kTimeoutMma; break; }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * kATile), b0 = smem_u32(sB + stage * kBTile);
#pragma unroll
                    for (int j = 0; j < BK / 32; ++j) {
                        // a k step of 32 moves a K-major tile's start by 32 bytes, an MN-major
                        // tile's by 32 rows of 128 bytes
                        const uint64_t ad = p.a_mn ? smem_desc_mn_sw128(a0 + 4096 * j) : smem_desc_sw128(a0 + 32 * j);
                        const uint64_t bd = p.b_mn ? smem_desc_mn_sw128(b0 + 4096 * j) : smem_desc_sw128(b0 + 32 * j);
                        mma_pair(tmem_base + static_cast<uint32_t>(acc * BN), ad, bd, idesc, (kb > 0 || j > 0));
                    }
                    commit_both(empty0 + 8 * stage);
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                if (fail) break;
                commit_both(tfull0 + 8 * acc);
                if (++acc == kAccBufs) { acc = 0; acc_phase ^= 1u; }
            }
            if (fail) *abort = 1;
            // every tensor-core operation issued has completed
            commit_local(drain_bar);
            if (!mbar_wait_drain(drain_bar, 0, p.wait_limit_ns)) fail |= kTimeoutDrain;
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int ew = warp - 2;
        const int quarter = warp & 3;
        const int cgrp = ew >> 2;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        int acc = 0;
        uint32_t acc_phase = 0;
        const float scale = __fmul_rn(__ldg(p.sa), __ldg(p.sb));
        for (int t = pair_id; t < tiles && !fail; t += pairs) {
            int mb, nb;
            tile_coords(t, p.tiles_m, p.tiles_n, mb, nb);
            const int row = mb * 2 * BM + static_cast<int>(rank) * BM + quarter * 32 + lane;
            const int col_base = nb * BN + cgrp * kColsPerWarp;
            if (p.num_kb > 0) {
                const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(tfull0 + 8 * acc, acc_phase, abort, p.wait_limit_ns));
                if (!ok) { fail = kTimeoutEpilogue; break; }
                tc_fence_after();
            }
            constexpr int kChunks = kColsPerWarp / 32;
            const uint32_t col_addr = tmem_base + lane_addr + static_cast<uint32_t>(acc * BN + cgrp * kColsPerWarp);
            uint32_t r0[32], r1[32];
            if (p.num_kb > 0) {
                tmem_ld32_async(col_addr, r0);
                tmem_wait32(r0);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) r0[i] = r1[i] = 0u;
            }
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                uint32_t (&cur)[32] = (c & 1) ? r1 : r0;
                uint32_t (&nxt)[32] = (c & 1) ? r0 : r1;
                if (p.num_kb > 0 && c + 1 < kChunks) tmem_ld32_async(col_addr + static_cast<uint32_t>(32 * (c + 1)), nxt);
                const int col0 = col_base + c * 32;
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(__uint_as_float(cur[i]), scale);
                if (p.bias) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (col0 + i < p.N) v[i] = __fadd_rn(v[i], load_bias<YT>(p.bias, col0 + i));
                }
                if (row < p.M && col0 < p.N) store_chunk<YT>(p, row, col0, v);
                if (p.num_kb > 0 && c + 1 < kChunks) tmem_wait32(nxt);
            }
            if (p.num_kb > 0) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) arrive_leader(tempty0 + 8 * acc);
                if (++acc == kAccBufs) { acc = 0; acc_phase ^= 1u; }
            }
        }
        if (fail && lane == 0) *abort = 1;
    }

    if (fail && p.status && lane == 0) atomicOr(p.status, fail);
    // neither CTA leaves (or frees TMEM) while the other may still signal its
    // barriers or the pair's MMAs may still write its TMEM
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace pair

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
    static EncodeTiled fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) !=
                cudaSuccess || q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<EncodeTiled>(f);
    }();
    return fn;
}

// 2-D map of a [rows][K] byte matrix, boxes of box_rows x 128 bytes, 128-byte
// swizzle; elements outside the matrix read as zero
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int box_rows) {
    EncodeTiled enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int YT, bool FINE, int BN_, int MT_>
cudaError_t launch_typed(const CUtensorMap& ma, const CUtensorMap& mb, const Params& p, uint32_t idesc,
                         cudaStream_t s) {
    auto kernel = scaled_mm_kernel<YT, FINE, BN_, MT_>;
    constexpr int kSmemBytes = Shape<BN_, MT_>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    const int tiles = p.tiles_m * p.tiles_n;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles < sm_count() ? tiles : sm_count()));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = FP8Q_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, ma, mb, p, idesc);
}

template <int BN_>
cudaError_t launch_dtype(bool fine, int yt, const CUtensorMap& ma, const CUtensorMap& mb, const Params& p,
                         uint32_t idesc, cudaStream_t s) {
    if (fine) {
        return yt == kF32 ? launch_typed<kF32, true, BN_, 128>(ma, mb, p, idesc, s)
             : yt == kF16 ? launch_typed<kF16, true, BN_, 128>(ma, mb, p, idesc, s)
                          : launch_typed<kBF16, true, BN_, 128>(ma, mb, p, idesc, s);
    }
    return yt == kF32 ? launch_typed<kF32, false, BN_, 128>(ma, mb, p, idesc, s)
         : yt == kF16 ? launch_typed<kF16, false, BN_, 128>(ma, mb, p, idesc, s)
                      : launch_typed<kBF16, false, BN_, 128>(ma, mb, p, idesc, s);
}

// per-tensor scales, 256 x 256 tiles
cudaError_t launch_tall(int yt, const CUtensorMap& ma, const CUtensorMap& mb, const Params& p, uint32_t idesc,
                        cudaStream_t s) {
    return yt == kF32 ? launch_typed<kF32, false, 256, 256>(ma, mb, p, idesc, s)
         : yt == kF16 ? launch_typed<kF16, false, 256, 256>(ma, mb, p, idesc, s)
                      : launch_typed<kBF16, false, 256, 256>(ma, mb, p, idesc, s);
}

// per-tensor scales, 256 x 256 tiles on CTA pairs: the grid is the pairs that
// fit at once (at most one per tile), two CTAs each
template <int YT>
cudaError_t launch_pair_typed(const CUtensorMap& ma, const CUtensorMap& mb, const Params& p, uint32_t idesc,
                              cudaStream_t s) {
    auto kernel = pair::scaled_mm_pair_kernel<YT>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pair::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pair::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = FP8Q_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cfg.gridDim = dim3(2);
    int fit = 0;
    if (cudaOccupancyMaxActiveClusters(&fit, kernel, &cfg) != cudaSuccess || fit < 1) fit = sm_count() / 2;
    const int tiles = p.tiles_m * p.tiles_n;
    const int pairs = tiles < fit ? tiles : fit;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    return cudaLaunchKernelEx(&cfg, kernel, ma, mb, p, idesc);
}

cudaError_t launch_pair(int yt, const CUtensorMap& ma, const CUtensorMap& mb, const Params& p, uint32_t idesc,
                        cudaStream_t s) {
    return yt == kF32 ? launch_pair_typed<kF32>(ma, mb, p, idesc, s)
         : yt == kF16 ? launch_pair_typed<kF16>(ma, mb, p, idesc, s)
                      : launch_pair_typed<kBF16>(ma, mb, p, idesc, s);
}

}  // namespace mm

fp8q_status launch_scaled_mm(const uint8_t* a, int fa, const uint8_t* b, int fb, int64_t M, int64_t N, int64_t K,
                             const float* sa, int sa_ld, const float* sb, int sb_ld, bool fine, const void* bias,
                             int yt, void* d, uint32_t* status, cudaStream_t s, int a_mn, int b_mn,
                             uint64_t wait_limit_ns, int stall_kb) {
    using namespace mm;
    // 128-wide tiles when a product of at most 128 rows would leave SMs idle
    const bool narrow = M <= BM && (N + 255) / 256 < sm_count();
    const int bn = narrow ? 128 : 256;
    // A product of fewer than 128 rows loads only its rows, rounded up to 16:
    // the MMA still multiplies 128 rows, and the rows past the box hold stale
    // shared memory, but output row m depends on row m of A alone and rows
    // at or past M are never stored.
    // (An MN-major A keeps its 128-wide box: its rows are k, its columns m.)
    // Per-tensor products take 256 x 256 tiles (two MMAs share each B tile)
    // when those tiles still fill nine tenths of the SMs.
    const int64_t tall_tiles = ((M + 2 * BM - 1) / (2 * BM)) * ((N + 255) / 256);
    const bool tall = !fine && !narrow && M >= 2 * BM && tall_tiles * 10 >= 9LL * sm_count();
    // 256 x 256 tiles on CTA pairs when those tiles give two CTAs each to nine
    // tenths of the SMs (the same tiles on one CTA each need twice as many)
    const bool pairs = FP8Q_PAIRS && !fine && !narrow && M >= 2 * BM && tall_tiles * 20 >= 9LL * sm_count();
    const int mt = (tall || pairs) ? 2 * BM : BM;
    const int a_rows = tall ? mt : (M >= BM || a_mn) ? BM : static_cast<int>((M + 15) / 16 * 16);
    CUtensorMap ma, mbm;
    memset(&ma, 0, sizeof(ma));
    memset(&mbm, 0, sizeof(mbm));
    if (K > 0 && pairs) {
        // each CTA of a pair loads 128 rows of A and 128 rows of B (MN-major: one
        // 128 k x 128-row box each)
        const bool ok_a = a_mn ? make_map(&ma, a, K, M, BK) : make_map(&ma, a, M, K, BM);
        const bool ok_b = b_mn ? make_map(&mbm, b, K, N, BK) : make_map(&mbm, b, N, K, pair::kHalfB);
        if (!ok_a || !ok_b) return FP8Q_ERR_CUDA;
    } else if (K > 0) {
        // K-major: [M][K] with boxes of rows x 128 k; MN-major: [K][M] with
        // boxes of 128 k x 128 m (B likewise, two boxes for 256 columns)
        const bool ok_a = a_mn ? make_map(&ma, a, K, M, BK) : make_map(&ma, a, M, K, a_rows);   // MN-major: 128-wide boxes
        const bool ok_b = b_mn ? make_map(&mbm, b, K, N, BK) : make_map(&mbm, b, N, K, bn);
        if (!ok_a || !ok_b) return FP8Q_ERR_CUDA;
    }
    Params p;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.num_kb = static_cast<int>((K + BK - 1) / BK);
    p.tiles_m = static_cast<int>((M + mt - 1) / mt);
    p.tiles_n = static_cast<int>((N + bn - 1) / bn);
    p.sa = sa;
    p.sb = sb;
    p.sa_ld = sa_ld;
    p.sb_ld = sb_ld;
    p.bias = bias;
    p.d = d;
    const int eb = yt == kF32 ? 4 : 2;
    p.vec_store = (reinterpret_cast<uintptr_t>(d) % 32 == 0) && ((N * eb) % 32 == 0);
    p.status = status;
    p.stage_tx = (a_rows + bn) * BK;
    p.a_mn = a_mn;
    p.b_mn = b_mn;
    p.wait_limit_ns = wait_limit_ns > 0 ? wait_limit_ns : kWaitLimitNs;
    p.stall_kb = stall_kb;
    const uint32_t idesc = instr_desc(fa, fb, bn, a_mn, b_mn);
    cudaError_t e;
    if (pairs) {
        // M 256 (128 rows per CTA), N 256
        const uint32_t pair_idesc = (1u << 4) | (static_cast<uint32_t>(fa) << 7) | (static_cast<uint32_t>(fb) << 10)
                                  | (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(b_mn) << 16)
                                  | (static_cast<uint32_t>(256 >> 3) << 17) | (static_cast<uint32_t>(256 >> 4) << 24);
        e = launch_pair(yt, ma, mbm, p, pair_idesc, s);
    } else if (narrow) e = launch_dtype<128>(fine, yt, ma, mbm, p, idesc, s);
    else if (tall) e = launch_tall(yt, ma, mbm, p, idesc, s);
    else e = launch_dtype<256>(fine, yt, ma, mbm, p, idesc, s);
    return cuda_status(e);
}

}  // namespace fp8q
