// gemm_blockwise.cu -- the consumer of the blockwise codes: an FP8 GEMM on
// the tcgen05 tensor cores with per-block scales applied in fp32.
//
// Mixed-precision handbook, section "FP8 training", closing notes: the
// matrix products take FP8 inputs with fp32 accumulation, and because an FP8
// tensor-core accumulator holds limited precision, every 128 products the
// partial sum is promoted to CUDA cores and accumulated there in fp32; the
// fine-grained scales (1x128 activations, 128x128 weights) are applied at that
// promotion.  Here
//     C[m][n] = sum over 128-wide K chunks c of
//               P_c[m][n] / (sa[m][c] * sb[n/128][c]),
//     P_c[m][n] = sum_{k in c} decode(A[m][k]) * decode(B[n][k]),
// with A [M, K] the 1x128-scaled codes (scales sa [M, K/128]) and B [N, K]
// the 128x128-scaled codes of a weight stored [out, in] (scales
// sb [N/128, K/128]); both scales are the quantizers' multipliers, so each
// promotion divides by them.
//
// The kernel is persistent: one CTA (or CTA pair) per SM (pair of SMs) walks
// the output tiles first, first + step, ..., numbered with the column tile
// fastest, so the CTAs running at one time share their rows of A and all of
// B in L2.  Per tile each CTA computes 128 rows x 256 columns of C (12 warps):
//   warp 0     TMA producer: per K chunk, a 128x128-byte box of A and the
//              box of B this CTA holds, into a ring of shared-memory stages
//              (128-byte swizzle, the layout the MMA descriptors name);
//   warp 1     allocates 512 TMEM columns (two 128x256 fp32 accumulators)
//              and issues the MMAs: per chunk, 4 x tcgen05.mma (K 32) into a
//              fresh accumulator, then commits to the stage's "empty" barrier
//              and the accumulator's "full" barrier;
//   warps 4-11 the promotion: each thread owns one row (its TMEM lane) and
//              128 columns; per chunk it loads its partial sums from TMEM,
//              frees the accumulator, and adds partial * 1/(sa * sb) into
//              128 fp32 registers.  The two accumulators alternate, so the
//              MMAs of chunk c+1 run while chunk c is promoted;
//   warps 2-3  idle (they complete the first warpgroup, whose registers go
//              to the promotion warpgroups).
// At the end of a tile each promotion thread writes its 128 results (fp32 or
// bf16).  Stages and accumulators are taken round-robin by a chunk count that
// runs on across tiles, so the producer prefetches the next tile and the MMAs
// start on it while the promotion warps store this one.
// Rows past M arrive as zeros from the copy engine and are not stored.
//
// B's scales come in two layouts (template BROW):
//   128  B in 128x128 blocks (a weight), sb [N/128, K/128]: one factor
//        1/(sa*sb) per row, chunk and column half;
//   1    B in 1x128 blocks along K (the weight gradient dW = dY^T X, whose
//        operands are both quantized along the tokens), sb [N, K/128]: warps
//        2-3 stage RN(1/sb) for the tile's 256 columns, 4 chunks per round
//        (one 16-byte load per column when the scales are aligned for it), in
//        an 8-slot shared-memory ring with its own barriers, and the
//        promotion multiplies each partial by RN(1/sa) and the column's
//        reciprocal, two elements per f32x2 instruction (56 control / 224
//        promotion registers).  Measured at 4096 x 7168 x 16384: 816 TF/s
//        with a scalar load per column and chunk, 874 with the 16-byte
//        loads, 901 with the packed arithmetic as well, 1056-1060 with the
//        row scales loaded ahead (FP8Q_GEMM_PREFETCH_SCALES).
// Two variants:
//   single CTA (M 128 x N 256 per MMA): the CTA loads A (16 KiB) and all of
//              B (32 KiB) per chunk, 4 stages;
//   CTA pair   (a cluster of 2, M 256 x N 256 per MMA): each CTA loads its
//              own 128 rows of A and one 128-row half of B (32 KiB per
//              chunk), and the tensor cores of the pair read the other half
//              from the peer -- a third less operand traffic per CTA for the
//              same work, and 6 stages.  The even CTA issues the MMAs; its
//              "full" barriers count both CTAs' copies, and both CTAs'
//              promotion warps release the accumulators to it.
// Measured on B200 (role timestamps): the MMA thread mostly waits for an
// accumulator to come back from the promotion, and each chunk's MMAs take
// about 0.6 us from issue to commit, so with two accumulators the chunks run
// nearly one at a time.  Four 128-column accumulator slots (N 128 MMAs) were
// slower; tiles cut into column halves (N 128) took as long per chunk as
// whole ones, so the chunk period is the hand-back latency, not the MMA work
// or the operand bytes; spinning waits changed nothing; a timing-only copy that accumulates
// all of K in one accumulator (no promotion) reaches about 2.2 PFLOP/s,
// bound there by the TMA operand delivery.
//
// Every barrier wait is bounded (1 s); a wait that runs out sets the
// wait-timeout bit of the device status word, and the CTA still waits
// (bounded) for its MMAs before it frees its tensor memory.

#include <algorithm>
#include <atomic>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "fp8q_device.cuh"
#include "fp8q_launch.h"
#include "launch_util.h"
#include "tensor_map.h"
#include "umma.cuh"

namespace fp8q {
namespace {

constexpr int kBM = 128;                  // rows of C per CTA (TMEM lanes)
constexpr int kBN = 256;                  // columns of C per CTA (MMA N)
constexpr int kBK = 128;                  // K chunk = one promotion = one stage
constexpr int kMmaK = 32;                 // K of one kind::f8f6f4 instruction
constexpr int kWarps = 12;                // 3 warpgroups: control, promotion x2
constexpr int kThreads = kWarps * 32;
constexpr int kABytes = kBM * kBK;        // 16 KiB
constexpr uint32_t kTmemCols = 2 * kBN;   // two accumulators
// Register split (setmaxnreg): the kernel launches at kLaunchRegs per thread;
// the control warpgroup gives registers back, the two promotion warpgroups
// take them.  The per-thread counts must add up to the launch total exactly
// (and per SM sub-partition: each holds one warp of every warpgroup), or an
// increase would never be granted.
constexpr int kLaunchRegs = 168;          // 65536 / 384 rounded down to a multiple of 8
#ifndef FP8Q_GEMM_B1_CONTROL_REGS
#define FP8Q_GEMM_B1_CONTROL_REGS 56
#endif
// 1x128 B moves registers from the promotion to the control warpgroup, whose
// warps 2-3 then stage the reciprocal column scales.
template <int BROW>
struct Split {
    static constexpr int kControlRegs = BROW == 1 ? FP8Q_GEMM_B1_CONTROL_REGS : 40;
    static constexpr int kPromoteRegs = (3 * kLaunchRegs - kControlRegs) / 2;
    static_assert(kControlRegs + 2 * kPromoteRegs == 3 * kLaunchRegs, "register split must equal the launch total");
    static_assert(kControlRegs % 8 == 0 && kPromoteRegs % 8 == 0, "setmaxnreg counts are multiples of 8");
};
static_assert(kLaunchRegs * kThreads <= 65536, "launch registers exceed the register file");

// The promotion loads its row's scales this many chunks ahead (0: in the chunk that uses them).
#ifndef FP8Q_GEMM_PREFETCH_SCALES
#define FP8Q_GEMM_PREFETCH_SCALES 2
#endif
// Tile order: -1 picks per call (row tile fastest when M < N), 0 column tile
// fastest, 1 row tile fastest.
#ifndef FP8Q_GEMM_RASTER
#define FP8Q_GEMM_RASTER -1
#endif
// 1x128 B: the fill's 16-byte scale loads, and packed f32x2 promotion arithmetic.
#ifndef FP8Q_GEMM_FILL_VEC4
#define FP8Q_GEMM_FILL_VEC4 1
#endif
#ifndef FP8Q_GEMM_PACKED_B1
#define FP8Q_GEMM_PACKED_B1 1
#endif

// B with 1x128 blocks (the weight-gradient operand) has a scale per column
// and chunk; two otherwise idle warps stage their reciprocals in a ring of
// kRbSlots chunks ahead of the promotion.
constexpr int kBarrierBytes = 512;       // shared memory reserved for the mbarriers
constexpr int kRbSlots = 8;
constexpr int kRbGroup = 4;               // chunks whose scales one fill round loads together
constexpr int kRbFillWarps = 2;           // warps 2 and 3
static_assert(kRbSlots % kRbGroup == 0 && kRbSlots >= 2 * kRbGroup, "the ring holds two fill rounds");

template <bool PAIR>
struct Cfg {
    static constexpr int kTileM = PAIR ? 2 * kBM : kBM;      // rows of C per tile (per pair)
    static constexpr int kBRows = PAIR ? kBN / 2 : kBN;      // rows of B this CTA loads
    static constexpr int kBBytes = kBRows * kBK;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = PAIR ? 6 : 4;
    static constexpr int kAccEmptyArrivals = PAIR ? 16 : 8;  // promotion warps releasing an accumulator
    static constexpr uint32_t kFullTx = PAIR ? 2 * kStageBytes : kStageBytes;  // bytes per "full" phase
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /* alignment */ + kBarrierBytes;
};
constexpr int kRbBytes = kRbSlots * kBN * 4;  // ring of per-column reciprocal B scales (1x128 B only)

template <int STAGES>
struct Barriers {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t mma_done;
    uint64_t rb_full[kRbSlots];
    uint64_t rb_empty[kRbSlots];
    uint32_t tmem_base;
};
static_assert(sizeof(Barriers<6>) <= kBarrierBytes, "barriers must fit their reserved bytes");
static_assert(sizeof(Barriers<4>) <= kBarrierBytes, "barriers must fit their reserved bytes");

// BROW: rows of a B scale block, 128 (128x128 blocks, sb [N/128, K/128]) or 1
// (1x128 blocks along K, sb [N, K/128]).
template <int OUT, bool PAIR, int BROW>
__global__ void __launch_bounds__(kThreads, 1)
k_gemm_blockwise(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 const float* __restrict__ sa, const float* __restrict__ sb, void* __restrict__ c, int64_t M,
                 int64_t N, int64_t K, uint32_t idesc, unsigned int* status, int row_fastest) {
    using C = Cfg<PAIR>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles_smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    auto* bars = reinterpret_cast<Barriers<C::kStages>*>(tiles_smem + C::kStages * C::kStageBytes);
    float* rb_ring = reinterpret_cast<float*>(tiles_smem + C::kStages * C::kStageBytes + kBarrierBytes);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? umma::cluster_ctarank() : 0u;  // 0: this CTA issues the MMAs
    // Persistent: this CTA (pair) takes tiles first, first + step, ...; a tile is
    // C::kTileM rows x kBN columns, numbered with the column tile fastest, or
    // with the row tile fastest when row_fastest is set (the host picks the
    // order in which the operand that every wave of tiles reads whole is the
    // smaller one, so that it stays in L2 from one wave to the next).
    const int64_t tiles_n = N / kBN;
    const int64_t tiles_m = (M + C::kTileM - 1) / C::kTileM;
    const int64_t tiles = tiles_m * tiles_n;
    auto tile_row = [&](int64_t t) { return row_fastest ? t % tiles_m : t / tiles_n; };
    auto tile_col = [&](int64_t t) { return row_fastest ? t / tiles_m : t % tiles_n; };
    const int64_t first = PAIR ? blockIdx.x / 2 : blockIdx.x;
    const int64_t step = PAIR ? gridDim.x / 2 : gridDim.x;
    const int nchunks = static_cast<int>(K / kBK);
    const int64_t kc_stride = K / kBK;  // scales per row of sa / sb

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            umma::mbar_init(&bars->full[s], 1);
            umma::mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            umma::mbar_init(&bars->acc_full[b], 1);
            umma::mbar_init(&bars->acc_empty[b], C::kAccEmptyArrivals);
        }
        umma::mbar_init(&bars->mma_done, 1);
        for (int r = 0; r < kRbSlots; ++r) {
            umma::mbar_init(&bars->rb_full[r], kRbFillWarps);
            umma::mbar_init(&bars->rb_empty[r], 8);  // this CTA's promotion warps
        }
        umma::fence_mbar_init();
    }
    if (warp == 1) {
        if (PAIR) umma::tmem_alloc_pair(&bars->tmem_base, kTmemCols);
        else umma::tmem_alloc(&bars->tmem_base, kTmemCols);
    }
    umma::fence_before_sync();
    __syncthreads();
    if (PAIR) umma::cluster_sync();  // the peer's barriers are initialised before any remote arrival
    umma::fence_after_sync();
    const uint32_t tmem = bars->tmem_base;
    pdl_enter();  // A, B and the scales may come from the previous kernel

    // Stages and accumulators are used round-robin by a chunk counter g that
    // runs on across tiles, so the producer prefetches the next tile and the
    // MMAs start on it while the promotion warps store this one.
    bool timed_out = false;
    if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(Split<BROW>::kControlRegs));
    if (warp == 0) {
        // ---- TMA producer ----------------------------------------------------
        if (lane == 0) {
            uint32_t g = 0;
            for (int64_t t = first; t < tiles && !timed_out; t += step) {
                const int m0 = static_cast<int>(tile_row(t) * C::kTileM + rank * kBM);
                const int n0 = static_cast<int>(tile_col(t) * kBN);
                for (int kc = 0; kc < nchunks; ++kc, ++g) {
                    const uint32_t s = g % C::kStages;
                    const uint32_t phase = (g / C::kStages) & 1u;
                    if (!umma::mbar_wait(&bars->empty[s], phase ^ 1u, kWaitLimitNs)) {
                        timed_out = true;
                        break;
                    }
                    uint8_t* stage = tiles_smem + s * C::kStageBytes;
                    if (PAIR) {
                        // both CTAs' copies complete on the even CTA's barrier, which
                        // expects the bytes of both
                        const uint32_t full0 = umma::mapa(umma::smem_u32(&bars->full[s]), 0);
                        if (rank == 0) umma::mbar_arrive_expect_tx(&bars->full[s], C::kFullTx);
                        umma::tma_load_2d_pair(stage, &map_a, full0, kc * kBK, m0);
                        umma::tma_load_2d_pair(stage + kABytes, &map_b, full0, kc * kBK,
                                               n0 + static_cast<int>(rank) * C::kBRows);
                    } else {
                        umma::mbar_arrive_expect_tx(&bars->full[s], C::kFullTx);
                        umma::tma_load_2d(stage, &map_a, &bars->full[s], kc * kBK, m0);
                        umma::tma_load_2d(stage + kABytes, &map_b, &bars->full[s], kc * kBK, n0);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer (the even CTA of a pair) -------------------------------
        if (lane == 0 && rank == 0) {
            const uint32_t peer_empty0 = PAIR ? umma::mapa(umma::smem_u32(&bars->empty[0]), 1) : 0u;
            const uint32_t peer_accf0 = PAIR ? umma::mapa(umma::smem_u32(&bars->acc_full[0]), 1) : 0u;
            uint32_t g = 0;
            for (int64_t t = first; t < tiles && !timed_out; t += step) {
                for (int kc = 0; kc < nchunks; ++kc, ++g) {
                    const uint32_t s = g % C::kStages;
                    const uint32_t phase = (g / C::kStages) & 1u;
                    const uint32_t buf = g & 1u;
                    const uint32_t acc_phase = (g >> 1) & 1u;
                    if (!umma::mbar_wait(&bars->acc_empty[buf], acc_phase ^ 1u, kWaitLimitNs) ||
                        !umma::mbar_wait(&bars->full[s], phase, kWaitLimitNs)) {
                        timed_out = true;
                        break;
                    }
                    umma::fence_after_sync();
                    const uint32_t a_addr = umma::smem_u32(tiles_smem + s * C::kStageBytes);
                    const uint64_t a_desc = umma::smem_desc_kmajor_sw128(a_addr);
                    const uint64_t b_desc = umma::smem_desc_kmajor_sw128(a_addr + kABytes);
                    const uint32_t d = tmem + buf * static_cast<uint32_t>(kBN);
#pragma unroll
                    for (int k = 0; k < kBK / kMmaK; ++k) {
                        // the next 32 bytes of K: start address + 32 bytes (2 in 16-byte units)
                        if (PAIR) umma::mma_f8f6f4_pair(d, a_desc + 2 * k, b_desc + 2 * k, idesc, k > 0);
                        else umma::mma_f8f6f4(d, a_desc + 2 * k, b_desc + 2 * k, idesc, k > 0);
                    }
                    if (PAIR) {
                        umma::commit_pair(umma::smem_u32(&bars->empty[s]));
                        umma::commit_pair(peer_empty0 + s * static_cast<uint32_t>(sizeof(uint64_t)));
                        umma::commit_pair(umma::smem_u32(&bars->acc_full[buf]));
                        umma::commit_pair(peer_accf0 + buf * static_cast<uint32_t>(sizeof(uint64_t)));
                    } else {
                        umma::commit(&bars->empty[s]);
                        umma::commit(&bars->acc_full[buf]);
                    }
                }
            }
            if (PAIR) umma::commit_pair(umma::smem_u32(&bars->mma_done));
            else umma::commit(&bars->mma_done);
            if (!umma::mbar_wait(&bars->mma_done, 0, kWaitLimitNs)) timed_out = true;
        }
    } else if (BROW == 1 && warp < 4) {
        // ---- reciprocal column scales of B (1x128 blocks), warps 2-3 ------------
        // A round loads the scales of up to kRbGroup chunks (16 loads in
        // flight per thread: the scales of a column are consecutive in K),
        // then waits for their ring slots and publishes them one by one.
        const int ft = (warp - 2) * 32 + lane;  // 0..63; columns ft + 64 i of the tile
        // A column's scales are consecutive in K: when every 4-chunk group starts on a 16-byte
        // boundary, a round takes them with one 16-byte load per column.
        const bool vec4 = FP8Q_GEMM_FILL_VEC4 && (kc_stride % kRbGroup) == 0 &&
                          (reinterpret_cast<uintptr_t>(sb) & 15u) == 0;
        uint32_t g = 0;
        for (int64_t t = first; t < tiles && !timed_out; t += step) {
            const float* sb_cols = sb + (tile_col(t) * kBN) * kc_stride;
            for (int kc0 = 0; kc0 < nchunks && !timed_out; kc0 += kRbGroup) {
                const int cnt = min(kRbGroup, nchunks - kc0);
                float v[kRbGroup][kBN / 64];
                if (vec4 && cnt == kRbGroup) {
                    static_assert(kRbGroup == 4, "one float4 per column and round");
#pragma unroll
                    for (int i = 0; i < kBN / 64; ++i) {
                        const float4 w = __ldg(reinterpret_cast<const float4*>(sb_cols + (ft + 64 * i) * kc_stride + kc0));
                        v[0][i] = w.x;
                        v[1][i] = w.y;
                        v[2][i] = w.z;
                        v[3][i] = w.w;
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < kRbGroup; ++u)
#pragma unroll
                        for (int i = 0; i < kBN / 64; ++i)
                            v[u][i] = (u < cnt) ? __ldg(sb_cols + (ft + 64 * i) * kc_stride + kc0 + u) : 1.0f;
                }
#pragma unroll
                for (int u = 0; u < kRbGroup; ++u) {
                    if (u >= cnt) break;
                    const uint32_t slot = (g + u) % kRbSlots;
                    const uint32_t phase = ((g + u) / kRbSlots) & 1u;
                    if (!umma::mbar_wait(&bars->rb_empty[slot], phase ^ 1u, kWaitLimitNs)) {
                        timed_out = true;
                        break;
                    }
                    float* rb = rb_ring + slot * kBN;
#pragma unroll
                    for (int i = 0; i < kBN / 64; ++i) rb[ft + 64 * i] = __frcp_rn(v[u][i]);
                    __syncwarp();
                    if (lane == 0) umma::mbar_arrive(&bars->rb_full[slot]);
                }
                g += static_cast<uint32_t>(cnt);
            }
        }
    } else if (warp >= 4) {
        // ---- promotion warps -------------------------------------------------
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(Split<BROW>::kPromoteRegs));
        const int quarter = warp & 3;            // TMEM lanes this warp may access
        const int half = (warp - 4) >> 2;        // column half of the tile
        const int row = quarter * 32 + lane;     // row within this CTA's 128 = TMEM lane
        const uint32_t acc_empty0 = PAIR ? umma::mapa(umma::smem_u32(&bars->acc_empty[0]), 0)
                                         : umma::smem_u32(&bars->acc_empty[0]);
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(half * 128);
        uint32_t g = 0;
        for (int64_t t = first; t < tiles && !timed_out; t += step) {
            const int64_t m = tile_row(t) * C::kTileM + rank * kBM + row;
            const int64_t col0 = tile_col(t) * kBN + half * 128;
            const float* sa_row = sa + (m < M ? m : 0) * kc_stride;
            const float* sb_row = sb + (BROW == 1 ? 0 : (col0 >> 7) * kc_stride);
            float acc[128];
#pragma unroll
            for (int j = 0; j < 128; ++j) acc[j] = 0.0f;
#if FP8Q_GEMM_PREFETCH_SCALES
            // this row's scales FP8Q_GEMM_PREFETCH_SCALES chunks ahead, so that their load latency is
            // not on the accumulator hand-back path
            constexpr int kAhead = FP8Q_GEMM_PREFETCH_SCALES;
            float sa_q[kAhead], sb_q[kAhead];
#pragma unroll
            for (int d = 0; d < kAhead; ++d) {
                sa_q[d] = (m < M && d < nchunks) ? __ldg(sa_row + d) : 1.0f;
                sb_q[d] = (BROW != 1 && m < M && d < nchunks) ? __ldg(sb_row + d) : 1.0f;
            }
#endif
            for (int kc = 0; kc < nchunks; ++kc, ++g) {
                const uint32_t buf = g & 1u;
                const uint32_t acc_phase = (g >> 1) & 1u;
                // 128x128 B: 1 / (sa * sb), the dequant factor of this chunk for this row and
                // column half.  1x128 B: 1 / sa here; 1 / sb per column from the ring.
#if FP8Q_GEMM_PREFETCH_SCALES
                const float sa_cur = sa_q[0], sb_cur = sb_q[0];
#pragma unroll
                for (int d = 0; d + 1 < kAhead; ++d) {
                    sa_q[d] = sa_q[d + 1];
                    sb_q[d] = sb_q[d + 1];
                }
                if (m < M && kc + kAhead < nchunks) {
                    sa_q[kAhead - 1] = __ldg(sa_row + kc + kAhead);
                    if (BROW != 1) sb_q[kAhead - 1] = __ldg(sb_row + kc + kAhead);
                }
                const float f = (m < M) ? (BROW == 1 ? __frcp_rn(sa_cur) : __frcp_rn(__fmul_rn(sa_cur, sb_cur)))
                                        : 0.0f;
#else
                const float f = (m < M) ? (BROW == 1 ? __frcp_rn(__ldg(sa_row + kc))
                                                     : __frcp_rn(__fmul_rn(__ldg(sa_row + kc), __ldg(sb_row + kc))))
                                        : 0.0f;
#endif
                const uint32_t slot = g % kRbSlots;
                if (!umma::mbar_wait(&bars->acc_full[buf], acc_phase, kWaitLimitNs)) {
                    timed_out = true;
                    break;
                }
                umma::fence_after_sync();
                const uint32_t tm = t_lane + buf * static_cast<uint32_t>(kBN);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float p[64];
                    umma::tmem_ld32(tm + h * 64, p);
                    umma::tmem_ld32(tm + h * 64 + 32, p + 32);
                    umma::wait_ld(p);
                    umma::hold_after_wait(p + 32);
                    if (h == 1) {
                        // every partial sum of this buffer is in registers: hand it back
                        umma::fence_before_sync();
                        __syncwarp();
                        if (lane == 0)
                            umma::mbar_arrive_cluster(acc_empty0 + buf * static_cast<uint32_t>(sizeof(uint64_t)));
                    }
                    if (BROW == 1) {
                        if (h == 0 && !umma::mbar_wait(&bars->rb_full[slot], (g / kRbSlots) & 1u, kWaitLimitNs)) {
                            timed_out = true;
                            break;
                        }
                        const float4* rb = reinterpret_cast<const float4*>(rb_ring + slot * kBN + half * 128 + h * 64);
#if FP8Q_GEMM_PACKED_B1
                        // the same two roundings per element, two elements per instruction:
                        // RN(p * f) (mul.rn.f32x2), then fma(that, 1/sb, acc) (fma.rn.f32x2)
                        const uint64_t f2 = f32x2(f, f);
#pragma unroll
                        for (int j4 = 0; j4 < 16; ++j4) {
                            const float4 r = rb[j4];
                            float* a = acc + h * 64 + 4 * j4;
                            const float2 lo = f32x2_split(fma_f32x2(mul_f32x2(f32x2(p[4 * j4], p[4 * j4 + 1]), f2),
                                                                    f32x2(r.x, r.y), f32x2(a[0], a[1])));
                            const float2 hi = f32x2_split(fma_f32x2(mul_f32x2(f32x2(p[4 * j4 + 2], p[4 * j4 + 3]), f2),
                                                                    f32x2(r.z, r.w), f32x2(a[2], a[3])));
                            a[0] = lo.x;
                            a[1] = lo.y;
                            a[2] = hi.x;
                            a[3] = hi.y;
                        }
#else
#pragma unroll
                        for (int j4 = 0; j4 < 16; ++j4) {
                            const float4 r = rb[j4];
                            acc[h * 64 + 4 * j4] = __fmaf_rn(__fmul_rn(p[4 * j4], f), r.x, acc[h * 64 + 4 * j4]);
                            acc[h * 64 + 4 * j4 + 1] =
                                __fmaf_rn(__fmul_rn(p[4 * j4 + 1], f), r.y, acc[h * 64 + 4 * j4 + 1]);
                            acc[h * 64 + 4 * j4 + 2] =
                                __fmaf_rn(__fmul_rn(p[4 * j4 + 2], f), r.z, acc[h * 64 + 4 * j4 + 2]);
                            acc[h * 64 + 4 * j4 + 3] =
                                __fmaf_rn(__fmul_rn(p[4 * j4 + 3], f), r.w, acc[h * 64 + 4 * j4 + 3]);
                        }
#endif
                        if (h == 1) {
                            __syncwarp();
                            if (lane == 0) umma::mbar_arrive(&bars->rb_empty[slot]);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 64; ++j) acc[h * 64 + j] = __fmaf_rn(p[j], f, acc[h * 64 + j]);
                    }
                }
                if (timed_out) break;
            }
            if (!timed_out && m < M) {
                if (OUT == 0) {
                    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(c) + m * N + col0);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        dst[j] = make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
                } else {
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(c) + m * N + col0);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        dst[j] = make_uint4(pack_bf16x2(acc[8 * j], acc[8 * j + 1]),
                                            pack_bf16x2(acc[8 * j + 2], acc[8 * j + 3]),
                                            pack_bf16x2(acc[8 * j + 4], acc[8 * j + 5]),
                                            pack_bf16x2(acc[8 * j + 6], acc[8 * j + 7]));
                }
            }
        }
    }
    if (timed_out) atomicOr(status, kStatusWaitTimeout);
    umma::fence_before_sync();
    if (__syncthreads_or(timed_out)) {
        // A wait ran out: give copies that may still be landing in this
        // CTA's shared memory time to finish (bounded) before it goes away.
        if (threadIdx.x == 0) {
            const uint64_t t0 = global_timer_ns();
            while (global_timer_ns() - t0 < 1000000ull) {
            }
        }
        __syncthreads();
    }
    // The even CTA's MMAs read the odd CTA's shared memory and write its
    // tensor memory: neither CTA frees or leaves before both are done.
    if (PAIR) umma::cluster_sync();
    if (warp == 1) {
        umma::fence_after_sync();
        if (PAIR) umma::tmem_dealloc_pair(tmem, kTmemCols);
        else umma::tmem_dealloc(tmem, kTmemCols);
    }
}

// [rows, K] bytes, K-major, boxes of box_rows x 128 bytes with the 128-byte
// swizzle; rows past the end read as zeros.
bool make_kmajor_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, uint32_t box_rows) {
    auto encode = tensor_map_encoder();
    if (encode == nullptr) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
    const cuuint32_t elem_strides[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, elem_strides,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int OUT, bool PAIR, int BROW>
cudaError_t launch_typed(const CUtensorMap& map_a, const CUtensorMap& map_b, const float* sa, const float* sb,
                         void* c, int64_t M, int64_t N, int64_t K, uint32_t idesc, unsigned int* status,
                         cudaStream_t st) {
    using C = Cfg<PAIR>;
    auto kern = k_gemm_blockwise<OUT, PAIR, BROW>;
    constexpr int kSmem = C::kSmemBytes + (BROW == 1 ? kRbBytes : 0);
    // The shared-memory opt-in, once per device (not inside a stream capture
    // on later calls).
    static std::atomic<bool> opted[128];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
    if (!opted[dev].load(std::memory_order_acquire)) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        opted[dev].store(true, std::memory_order_release);
    }
    const int64_t tiles = ((M + C::kTileM - 1) / C::kTileM) * (N / kBN);
    if (tiles == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
#if FP8Q_PDL
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
#endif
    if (PAIR) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 2;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    // Persistent grid: as many CTAs (pairs) as fit on the device at once (one
    // per SM), never more than there are tiles.
    static std::atomic<int> resident[128];
    int units = resident[dev].load(std::memory_order_acquire);
    if (units <= 0) {
        units = PAIR ? device_sm_count() / 2 : device_sm_count();
        if (PAIR) {
            int clusters = 0;
            cfg.gridDim = dim3(2 * static_cast<unsigned>(units));
            const cudaError_t oe = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
            if (oe != cudaSuccess) (void)cudaGetLastError();  // keep the device-count estimate
            else if (clusters > 0) units = std::min(units, clusters);
        }
        resident[dev].store(std::max(units, 1), std::memory_order_release);
    }
    const int64_t ctas = std::min<int64_t>(tiles, units) * (PAIR ? 2 : 1);
    cfg.gridDim = dim3(static_cast<unsigned>(ctas));
#if FP8Q_GEMM_RASTER < 0
    const int row_fastest = M < N ? 1 : 0;  // each wave reads all of A (row fastest) or all of B
#else
    const int row_fastest = FP8Q_GEMM_RASTER;
#endif
    const cudaError_t e =
        cudaLaunchKernelEx(&cfg, kern, map_a, map_b, sa, sb, c, M, N, K, idesc, status, row_fastest);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

bool gemm_blockwise_supported() { return tensor_map_encoder() != nullptr; }

cudaError_t launch_gemm_blockwise(const uint8_t* a, const float* sa, int a_fmt, const uint8_t* b, const float* sb,
                                  int b_block_rows, int b_fmt, int64_t M, int64_t N, int64_t K, void* c, int c_dtype,
                                  cudaStream_t st) {
    // A pair pays off once there are two row tiles to share B between.
    const bool pair = M > kBM;
    CUtensorMap map_a, map_b;
    if (!make_kmajor_map(&map_a, a, M, K, kBM) || !make_kmajor_map(&map_b, b, N, K, pair ? kBN / 2 : kBN))
        return cudaErrorInvalidValue;
    unsigned int* status = device_status_word();
    if (status == nullptr) return cudaErrorInvalidValue;
    const uint32_t idesc = umma::instr_desc_f8f6f4(a_fmt, b_fmt, pair ? 2 * kBM : kBM, kBN);
#define FP8Q_GEMM_LAUNCH(OUT, PAIR, BROW) \
    launch_typed<OUT, PAIR, BROW>(map_a, map_b, sa, sb, c, M, N, K, idesc, status, st)
    if (b_block_rows == 1) {
        if (pair) return c_dtype == 0 ? FP8Q_GEMM_LAUNCH(0, true, 1) : FP8Q_GEMM_LAUNCH(1, true, 1);
        return c_dtype == 0 ? FP8Q_GEMM_LAUNCH(0, false, 1) : FP8Q_GEMM_LAUNCH(1, false, 1);
    }
    if (pair) return c_dtype == 0 ? FP8Q_GEMM_LAUNCH(0, true, 128) : FP8Q_GEMM_LAUNCH(1, true, 128);
    return c_dtype == 0 ? FP8Q_GEMM_LAUNCH(0, false, 128) : FP8Q_GEMM_LAUNCH(1, false, 128);
#undef FP8Q_GEMM_LAUNCH
}

}  // namespace fp8q
