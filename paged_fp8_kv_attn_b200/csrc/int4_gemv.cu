// int4_gemv.cu -- decode-time INT4 weight dequantisation GEMV for sm_100a.
//
// Source pages: "大模型推理优化：量化、压缩与安全验证", section "压缩模型权重"
// (weights stored as 4-bit integers and expanded back to floating point
// before the multiply; decode streams every weight from memory once per
// token, so fewer bytes mean faster tokens); siami.tw editorial, section
// "模型權重壓縮：GLM 5.2 從 705 GB 縮到 421 GB" (Table 2: FP8 vs INT4 weight
// decode throughput against concurrency); remio.ai commentary, section
// "GLM 权重压缩改变了阶段权衡".  The pages fix no format; the one here:
// signed two's complement codes in tiles of 128 rows x 256 columns (16 KiB,
// row-major, two codes per byte with the even column in the low nibble;
// tiles ordered by row block, then column block), one bf16 scale per
// 128-column group of a row stored [row block][group][row in block], and
// y[b][j] = bf16(sum_i x[b][i] * q[j][i] * scale(j, i / 128)).  The tiles
// make each pipeline stage one contiguous 16 KiB read: with row-major rows
// a stage would gather 128 separate 128-byte pieces 4 KiB apart.
//
// Design:
//  * One CTA per 128 weight rows (output features) and slice of up to 32
//    batch rows (two slices above 32, as adjacent CTAs that read the same
//    codes at the same time, the second copy from L2).  The last warp (the producer)
//    streams the rows' codes (16 KiB per 256 columns), the matching x
//    columns of the whole batch and the two groups' scales into a ring of
//    shared-memory stages with 2-D TMA loads on full/empty mbarriers; the
//    first stages' codes are prefetched into L2 before the grid-dependency
//    wait.  Warps 0-3 each own 32 rows (two m16 blocks).
//  * Math on tensor cores: m16n8k16 bf16 MMAs, weight rows as M, the batch
//    as N in blocks of 8 (kNB blocks; padding rows of x are zero-filled by
//    TMA).  A code pair becomes bf16x2 (136 + q_lo, 136 + q_hi) by moving
//    each nibble into the low mantissa bits of 128.0 with its sign bit
//    flipped (one PRMT + one LOP3), then (q_lo, q_hi) exactly by one bf16x2
//    FMA with -136.  Codes are integers, so each 128-column group is
//    accumulated unscaled in fp32 and then added to the output accumulator
//    times the row's group scale: no bf16 rounding of q * scale.
//  * Column order inside a 64-column block: thread c of a quad feeds MMA
//    columns 2c, 2c+1 (and 2c+8, 2c+9) of k-step j from physical columns
//    16c + 4j + {0, 1} ({2, 3}); the same map picks x, so every dot product
//    is unchanged while each thread reads 8 contiguous code bytes and 32
//    contiguous x bytes per block.
//  * Bank conflicts: TMA writes 128-byte rows with the 128-byte swizzle
//    (16-byte unit XOR row mod 8).  A half-warp's 8-byte code loads touch
//    two adjacent units in each of 4 rows; MMA row g reads tile row
//    2 (g mod 4) + g / 4 of its 8-row half, so those 4 rows have row mod 8 in
//    {0, 2, 4, 6} (or the odd ones) and the 8 units fall in distinct banks.
#include "device.cuh"
#include "internal.h"

namespace pkv {

template <int kNB, int kCW>
struct GemvCfg {
    static constexpr int kWBytes = kGemvRows * kGemvKTile / 2;     // codes of a stage: 16 KiB
    static constexpr int kXBoxBytes = kNB * 8 * 128;               // x rows x 64 columns (bf16)
    static constexpr int kXBytes = (kGemvKTile / 64) * kXBoxBytes;
    static constexpr int kSBytes = (kGemvKTile / kGemvGroup) * kGemvRows * 2;
    static constexpr int kStageBytes = (kWBytes + kXBytes + kSBytes + 1023) / 1024 * 1024;
    // two CTAs per SM in every variant; the depth fills what is left
    static constexpr int kStages = kNB <= 2 ? 4 : 3;
    static constexpr int kThreads = 32 * (kCW + 1);                // consumer warps + producer
    static constexpr int kMB = kGemvRows / 16 / kCW;               // m16 blocks per consumer warp
    static constexpr int kBarOff = kStages * kStageBytes;
    static constexpr int kSmemBytes = kBarOff + 2 * kStages * 8 + 16 + 1024;   // + alignment slack
    static_assert(kNB == 1 || kNB == 2 || kNB == 4, "batch blocks");
    static_assert(kCW == 4 || kCW == 8, "consumer warps");
};

// bf16x2 (q_lo, q_hi) of the two codes in byte `b` of w (w4 = w >> 4).
__device__ __forceinline__ uint32_t int4x2_to_bf16x2(uint32_t w, uint32_t w4, uint32_t b) {
    // result byte 0 = byte b of w (low nibble q_lo), byte 2 = byte b of w4 (q_hi)
    const uint32_t t = prmt(w, w4, b | (b << 4) | ((b + 4) << 8) | ((b + 4) << 12));
    uint32_t v;   // (t & 0x000F000F) ^ 0x43084308: mantissa = nibble ^ 8 = q + 8 under 2^7
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(v) : "r"(t), "r"(0x000F000Fu), "r"(0x43084308u));
    uint32_t r;   // (136 + q) * 1 - 136, exact in bf16
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(v), "r"(0x3F803F80u), "r"(0xC308C308u));
    return r;
}

__device__ __forceinline__ bool gemv_wait(uint64_t* bar, uint32_t parity, volatile int* failed,
                                          uint32_t* status) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*failed) return false;
    if (mbar_wait(bar, parity)) return true;
    *failed = 1;
    if (status != nullptr) atomicOr(status, 1u);
    return false;
}

template <int kNB, int kCW>
__global__ void __launch_bounds__(GemvCfg<kNB, kCW>::kThreads, 2)
int4_gemv_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                 const __grid_constant__ CUtensorMap tmap_s, const GemvArgs a) {
    using C = GemvCfg<kNB, kCW>;
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
    // CTA -> (row tile, batch slice of 8 kNB rows); the slices of one tile are
    // adjacent CTAs, so they run together and share the tile's codes in L2
    const int slices = (a.batch + 8 * kNB - 1) / (8 * kNB);
    const int row0 = (blockIdx.x / slices) * kGemvRows;
    const int b0 = (blockIdx.x % slices) * 8 * kNB;
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
                    tma_load_2d(base + C::kWBytes + i * C::kXBoxBytes, &tmap_x, t * kGemvKTile + i * 64, b0,
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
                        const uint32_t by = 2 * (j & 1);
                        const uint32_t a0 = int4x2_to_bf16x2(lo, lo >> 4, by);
                        const uint32_t a2 = int4x2_to_bf16x2(lo, lo >> 4, by + 1);
                        const uint32_t a1 = int4x2_to_bf16x2(hi, hi >> 4, by);
                        const uint32_t a3 = int4x2_to_bf16x2(hi, hi >> 4, by + 1);
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
                const int b = b0 + 8 * nb + 2 * c + (i & 1);
                const int nn = nlo + ((i & 2) ? 8 : 0);
                if (b < a.batch) a.y[static_cast<int64_t>(b) * a.n + nn] = f32_to_bf16_bits(acc[m][nb][i]);
            }
    }
}

// Consumer warps per CTA: four warps of 32 rows (eight warps of 16 rows
// measured the same on B200 and spill at batch 32).
template <int kNB>
struct GemvVariant {
    static constexpr int kCW = 4;
    using Cfg = GemvCfg<kNB, kCW>;
};

int gemv_batch_blocks(int batch) {
    const int nb = (batch + 7) / 8;
    return nb <= 1 ? 1 : (nb <= 2 ? 2 : 4);
}

#define PKV_GEMV_DISPATCH(nb, EXPR) \
    switch (nb) {                    \
        case 1: { constexpr int NB = 1; EXPR; } \
        case 2: { constexpr int NB = 2; EXPR; } \
        case 4: { constexpr int NB = 4; EXPR; } \
        default: return cudaErrorInvalidValue; \
    }

cudaError_t gemv_set_smem_attr(int nb) {
    PKV_GEMV_DISPATCH(nb, return cudaFuncSetAttribute(
                              int4_gemv_kernel<NB, GemvVariant<NB>::kCW>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              GemvVariant<NB>::Cfg::kSmemBytes))
}

size_t gemv_smem_bytes(int nb) {
    switch (nb) {
        case 1: return GemvVariant<1>::Cfg::kSmemBytes;
        case 2: return GemvVariant<2>::Cfg::kSmemBytes;
        case 4: return GemvVariant<4>::Cfg::kSmemBytes;
        default: return 0;
    }
}

cudaError_t launch_int4_gemv(int nb, cudaStream_t stream, const CUtensorMap& tmap_w,
                             const CUtensorMap& tmap_x, const CUtensorMap& tmap_s, const GemvArgs& args) {
    const int slices = (args.batch + 8 * nb - 1) / (8 * nb);
    PKV_GEMV_DISPATCH(nb, {
        PdlLaunch l(dim3(args.n / kGemvRows * slices), dim3(GemvVariant<NB>::Cfg::kThreads),
                    GemvVariant<NB>::Cfg::kSmemBytes, stream);
        return cudaLaunchKernelEx(&l.cfg, int4_gemv_kernel<NB, GemvVariant<NB>::kCW>, tmap_w, tmap_x,
                                  tmap_s, args);
    })
}

}  // namespace pkv
