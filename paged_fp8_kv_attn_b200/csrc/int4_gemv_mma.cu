// int4_gemv_mma.cu -- INT4 weight dequantisation GEMV for batches of at most
// 16, on the warp-level tensor-core path (mma.sync m16n8k16).
//
// Source pages and format: as in int4_gemv.cu ("压缩模型权重"; siami.tw,
// "模型權重壓縮：GLM 5.2 從 705 GB 縮到 421 GB", Table 2; remio.ai, "GLM 权重压缩
// 改变了阶段权衡"): tiled signed 4-bit codes, 8-column words with the even
// columns in the low half-word, bf16 group scales, fp32 accumulation.
//
// Why a second kernel: at decode batch sizes the tensor-core tile is thin.
// A tcgen05.mma of M = 128 rows and K = 16 takes about the same time for
// N = 16 as for N = 64 (measured on B200: roughly 100 cycles per
// instruction), which caps the tcgen05 kernel near 2.7 TB/s of codes,
// whereas m16n8k16 MMAs cost in proportion to N and keep up with the code
// stream for N <= 16.  Above 16 rows the tcgen05 kernel is faster.
//
// Design:
//  * One CTA per 128 weight rows; warp 4 streams each 256-column code tile
//    (16 KiB, one contiguous TMA box), x for the batch (8 or 16 rows,
//    zero-filled) and the two groups' scales into a ring of stages; warps
//    0-3 own 32 rows each.
//  * m16n8k16 bf16 MMAs with weight rows as M and the batch as N.  A code
//    pair becomes bf16x2 (q_even, q_odd) with one shift, one LOP3 (the
//    offset-binary nibbles into the mantissas of 128.0) and one bf16x2 FMA
//    (minus 136).  Each 128-column group is summed unscaled in fp32 and then
//    added to the output accumulator times the row's group scale.
//  * Column order inside a 64-column block: thread c of a quad feeds MMA
//    columns 2c, 2c+1 (and 2c+8, 2c+9) of k-step j from physical columns
//    16c + 4j + {0, 1} ({2, 3}); the same map picks x, so every dot product
//    is unchanged while each thread reads 8 contiguous code bytes and 32
//    contiguous x bytes per block.
//  * Bank conflicts: TMA writes 128-byte rows with the 128-byte swizzle.  A
//    half-warp's 8-byte code loads touch two adjacent units in each of 4
//    rows; MMA row g reads tile row 2 (g mod 4) + g / 4 of its 8-row half,
//    so those 4 rows have row mod 8 in {0, 2, 4, 6} (or the odd ones) and
//    the 8 units fall in distinct banks.
#include "device.cuh"
#include "internal.h"

namespace pkv {

template <int kNB, int kCW>
struct MmaGemvCfg {
    static constexpr int kWBytes = kGemvRows * kGemvKTile / 2;     // codes of a stage: 16 KiB
    static constexpr int kXBoxBytes = kNB * 8 * 128;               // x rows x 64 columns (bf16)
    static constexpr int kXBytes = (kGemvKTile / 64) * kXBoxBytes;
    static constexpr int kSBytes = (kGemvKTile / kGemvGroup) * kGemvRows * 2;
    static constexpr int kStageBytes = (kWBytes + kXBytes + kSBytes + 1023) / 1024 * 1024;
    // two CTAs per SM in every variant; the depth fills what is left
    static constexpr int kStages = 4;
    static constexpr int kThreads = 32 * (kCW + 1);                // consumer warps + producer
    static constexpr int kMB = kGemvRows / 16 / kCW;               // m16 blocks per consumer warp
    static constexpr int kBarOff = kStages * kStageBytes;
    static constexpr int kSmemBytes = kBarOff + 2 * kStages * 8 + 16 + 1024;   // + alignment slack
    static_assert(kNB == 1 || kNB == 2, "batch blocks");
    static_assert(kCW == 4 || kCW == 8, "consumer warps");
};

template <int kNB, int kCW>
__global__ void __launch_bounds__(MmaGemvCfg<kNB, kCW>::kThreads, 2)
int4_gemv_mma_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                 const __grid_constant__ CUtensorMap tmap_s, const GemvArgs a) {
    using C = MmaGemvCfg<kNB, kCW>;
    constexpr int S = C::kStages;
    constexpr int MB = C::kMB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* empty_bar = full_bar + S;
    volatile int* failed = reinterpret_cast<volatile int*>(empty_bar + S);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int row0 = blockIdx.x * kGemvRows;
    const int KT = a.k / kGemvKTile;

    launch_dependents();
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kCW);
        }
        *failed = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == kCW) {
        // ================= producer =================
        if (lane == 0) {
            prefetch_tensormap(&tmap_w);
            prefetch_tensormap(&tmap_x);
            prefetch_tensormap(&tmap_s);
            // the weights are not written by preceding kernels: start early
            const int tile0 = (row0 / kGemvRows) * KT;     // first code tile of the row block
            for (int t = 0; t < S && t < KT; ++t) tma_prefetch_l2_2d(&tmap_w, 0, (tile0 + t) * kGemvRows);
            grid_dependency_wait();
            for (int t = 0; t < KT; ++t) {
                const int stage = t % S;
                if (t >= S) gemv_wait(&empty_bar[stage], ((t / S) + 1) & 1, failed, a.status);
                const uint32_t base = smem_addr(smem + stage * C::kStageBytes);
                mbar_arrive_expect_tx(&full_bar[stage], C::kWBytes + C::kXBytes + C::kSBytes);
                tma_load_2d(base, &tmap_w, 0, (tile0 + t) * kGemvRows, &full_bar[stage]);
#pragma unroll
                for (int i = 0; i < kGemvKTile / 64; ++i)
                    tma_load_2d(base + C::kWBytes + i * C::kXBoxBytes, &tmap_x, t * kGemvKTile + i * 64, 0,
                                &full_bar[stage]);
                tma_load_2d(base + C::kWBytes + C::kXBytes, &tmap_s, 0,
                            (row0 / kGemvRows) * (a.k / kGemvGroup) + t * (kGemvKTile / kGemvGroup),
                            &full_bar[stage]);
            }
        }
        return;
    }

    // ================= consumers =================
    const int g = lane >> 2;
    const int c = lane & 3;
    const int pg = ((g & 3) << 1) | (g >> 2);      // tile row of MMA row g in its 8-row half
    const int rw = 16 * MB * warp;                   // first tile row of this warp

    float acc[MB][kNB][4];
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int nb = 0; nb < kNB; ++nb) acc[mb][nb][0] = acc[mb][nb][1] = acc[mb][nb][2] = acc[mb][nb][3] = 0.f;

    for (int t = 0; t < KT; ++t) {
        const int stage = t % S;
        gemv_wait(&full_bar[stage], (t / S) & 1, failed, a.status);
        const uint32_t wbase = smem_addr(smem + stage * C::kStageBytes);
        const uint32_t xbase = wbase + C::kWBytes;
        const uint16_t* sbase =
            reinterpret_cast<const uint16_t*>(smem + stage * C::kStageBytes + C::kWBytes + C::kXBytes);
#pragma unroll
        for (int grp = 0; grp < kGemvKTile / kGemvGroup; ++grp) {
            float gacc[MB][kNB][4];
#pragma unroll
            for (int m = 0; m < MB; ++m)
#pragma unroll
                for (int nb = 0; nb < kNB; ++nb)
                    gacc[m][nb][0] = gacc[m][nb][1] = gacc[m][nb][2] = gacc[m][nb][3] = 0.f;
#pragma unroll
            for (int bb = 0; bb < kGemvGroup / 64; ++bb) {
                const int blk = grp * (kGemvGroup / 64) + bb;       // 64-column block of the tile
                // codes: 8 bytes (columns 64 blk + 16c .. +15) of rows rlo and rlo + 8
                uint2 wl[MB], wh[MB];
#pragma unroll
                for (int m = 0; m < MB; ++m) {
                    const int rlo = rw + 16 * m + pg;
                    wl[m] = lds64(wbase + swz<128, 128>(rlo, 32 * blk + 8 * c));
                    wh[m] = lds64(wbase + swz<128, 128>(rlo + 8, 32 * blk + 8 * c));
                }
                const uint32_t xbox = xbase + blk * C::kXBoxBytes;
                uint4 xv[kNB];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    // x: columns 64 blk + 16c + 8 (j/2) .. +7 of batch row 8 nb + g
                    if ((j & 1) == 0) {
#pragma unroll
                        for (int nb = 0; nb < kNB; ++nb)
                            xv[nb] = lds128(xbox + swz<128, 128>(8 * nb + g, 32 * c + 16 * (j >> 1)));
                    }
#pragma unroll
                    for (int m = 0; m < MB; ++m) {
                        const uint32_t lo = (j < 2) ? wl[m].x : wl[m].y;
                        const uint32_t hi = (j < 2) ? wh[m].x : wh[m].y;
                        // a word holds 8 columns; pair p = columns (2p, 2p + 1) sits at bit 4p
                        const uint32_t sh = 8 * (j & 1);
                        const uint32_t a0 = int4_pair_to_bf16x2(lo >> sh);
                        const uint32_t a2 = int4_pair_to_bf16x2(lo >> (sh + 4));
                        const uint32_t a1 = int4_pair_to_bf16x2(hi >> sh);
                        const uint32_t a3 = int4_pair_to_bf16x2(hi >> (sh + 4));
#pragma unroll
                        for (int nb = 0; nb < kNB; ++nb)
                            mma_bf16(gacc[m][nb], a0, a1, a2, a3, (j & 1) ? xv[nb].z : xv[nb].x,
                                     (j & 1) ? xv[nb].w : xv[nb].y);
                    }
                }
            }
            // scale the group's sums by the rows' scales (rows rlo: c0, c1; rlo + 8: c2, c3)
#pragma unroll
            for (int m = 0; m < MB; ++m) {
                const int rlo = rw + 16 * m + pg;
                const float s_lo = bf16_bits_to_f32(sbase[grp * kGemvRows + rlo]);
                const float s_hi = bf16_bits_to_f32(sbase[grp * kGemvRows + rlo + 8]);
#pragma unroll
                for (int nb = 0; nb < kNB; ++nb) {
                    acc[m][nb][0] = fmaf(s_lo, gacc[m][nb][0], acc[m][nb][0]);
                    acc[m][nb][1] = fmaf(s_lo, gacc[m][nb][1], acc[m][nb][1]);
                    acc[m][nb][2] = fmaf(s_hi, gacc[m][nb][2], acc[m][nb][2]);
                    acc[m][nb][3] = fmaf(s_hi, gacc[m][nb][3], acc[m][nb][3]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[stage]);
    }

    // y[b][n]: accumulator (row, col) = (weight row, batch row)
    grid_dependency_wait();
#pragma unroll
    for (int m = 0; m < MB; ++m) {
        const int nlo = row0 + rw + 16 * m + pg;
#pragma unroll
        for (int nb = 0; nb < kNB; ++nb)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int b = 8 * nb + 2 * c + (i & 1);
                const int nn = nlo + ((i & 2) ? 8 : 0);
                if (b < a.batch) a.y[static_cast<int64_t>(b) * a.n + nn] = f32_to_bf16_bits(acc[m][nb][i]);
            }
    }
}

// Consumer warps per CTA: four warps of 32 rows (eight warps of 16 rows
// measured the same on B200 and spill at batch 32).
template <int kNB>
struct MmaGemvVariant {
    static constexpr int kCW = 4;
    using Cfg = MmaGemvCfg<kNB, kCW>;
};

int gemv_mma_batch_blocks(int batch) { return batch <= 8 ? 1 : 2; }

#define PKV_GEMV_MMA_DISPATCH(nb, EXPR) \
    switch (nb) {                        \
        case 1: { constexpr int NB = 1; EXPR; } \
        case 2: { constexpr int NB = 2; EXPR; } \
        default: return cudaErrorInvalidValue; \
    }

cudaError_t gemv_mma_set_smem_attr(int nb) {
    PKV_GEMV_MMA_DISPATCH(nb, return cudaFuncSetAttribute(
                                  int4_gemv_mma_kernel<NB, MmaGemvVariant<NB>::kCW>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  MmaGemvVariant<NB>::Cfg::kSmemBytes))
}

cudaError_t launch_int4_gemv_mma(int nb, cudaStream_t stream, const CUtensorMap& tmap_w,
                                 const CUtensorMap& tmap_x, const CUtensorMap& tmap_s,
                                 const GemvArgs& args) {
    PKV_GEMV_MMA_DISPATCH(nb, {
        PdlLaunch l(dim3(args.n / kGemvRows), dim3(MmaGemvVariant<NB>::Cfg::kThreads),
                    MmaGemvVariant<NB>::Cfg::kSmemBytes, stream);
        return cudaLaunchKernelEx(&l.cfg, int4_gemv_mma_kernel<NB, MmaGemvVariant<NB>::kCW>, tmap_w,
                                  tmap_x, tmap_s, args);
    })
}

}  // namespace pkv
