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
// row-major, tiles ordered by row block then column block); each 32-bit
// word of a row holds 8 consecutive columns, the even ones in the low
// half-word and the odd ones in the high half-word; one bf16 scale per
// 128-column group of a row stored [row block][group][row in block]; and
// y[b][j] = bf16(sum_i x[b][i] * q[j][i] * scale(j, i / 128)).
//
// Design (tcgen05 / tensor memory):
//  * Used for batches above 16 (int4_gemv_mma.cu covers smaller ones).
//  * One half-CTA per 128 weight rows: a CTA holds two independent halves
//    (warps 0-5 and 6-11), each with its own shared memory, barriers and
//    tensor-memory columns (a CTA that allocates tensor memory is the only
//    one on its SM).  Below, warp numbers are within a half.  Warp 4
//    streams, with 2-D TMA loads, the rows' codes (one contiguous 16 KiB
//    tile per 256 columns) and the two
//    groups' scales into one ring of shared-memory stages (lane 0), and the
//    matching columns of x for the whole batch (zero-filled up to N = 32 or 64
//    rows) into a second ring (lane 1); the first code tiles are
//    prefetched into L2 before the grid-dependency wait.
//  * Warps 0-3 convert: each owns the 32 rows of its tensor-memory lane
//    quarter (the warp's index in the CTA mod 4; thread = row = lane).  Per
//    128-column group a thread expands its row's 128 codes to bf16 in
//    registers (per pair of columns: one shift, one LOP3 that puts the two
//    offset-binary nibbles into the mantissas of 128.0, one bf16x2 FMA that
//    subtracts 136) and writes them to a tensor-memory A buffer with
//    tcgen05.st.
//  * Warp 5 issues the tensor-core work: per group eight
//    tcgen05.mma.kind::f16 (M = 128 rows, N = batch, K = 16) with A from
//    tensor memory and x (B, K-major, 128-byte swizzle) straight from the
//    TMA tile, accumulating the group's unscaled sums in a tensor-memory
//    accumulator; tcgen05.commit signals the converter warps and, after a
//    stage's last group, frees the stage.
//  * A and the accumulator are double-buffered by group parity, so a group's
//    expansion overlaps the previous group's MMAs.  Each thread reads its
//    row of a finished group's accumulator (tcgen05.ld) and adds it times
//    the row's group scale to fp32 registers: the codes are exact in bf16,
//    the products exact in fp32, and nothing is rounded to bf16 before the
//    final output.
//  * Every mbarrier wait is bounded; the tensor memory is always freed.
#include "device.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace pkv {

template <int kN>
struct GemvCfg {
    // Two rings.  Code ring: a 16 KiB code tile and the two groups' scales
    // per 256 columns, freed as soon as the converter warps hold them in
    // registers.  x ring: the batch's 256 columns of x, freed by the MMA
    // commit.  Splitting them keeps a code stage's lifetime short (TMA
    // latency plus a register copy) instead of TMA + expansion + MMA.
    static constexpr int kWBytes = kGemvRows * kGemvKTile / 2;      // 16 KiB
    static constexpr int kSBytes = (kGemvKTile / kGemvGroup) * kGemvRows * 2;
    static constexpr int kWStageBytes = (kWBytes + kSBytes + 1023) / 1024 * 1024;
    static constexpr int kXBoxBytes = kN * 128;                     // kN rows x 64 columns (bf16)
    static constexpr int kXStageBytes = (kGemvKTile / 64) * kXBoxBytes;
    // two halves per CTA; the depths fill what is left of the shared memory
    static constexpr int kXStages = 2;
    static constexpr int kWStages = kN == 32 ? 4 : 2;
    static constexpr int kXOff = kWStages * kWStageBytes;
    // converter warps: kSplit per tensor-memory lane quarter, each taking
    // 1 / kSplit of a group's columns and of the batch columns (one per
    // quarter measured faster than two: the MMA issue is the bottleneck);
    // then the TMA warp and the MMA warp
    static constexpr int kSplit = 1;
    static constexpr int kConverters = 4 * kSplit;
    static constexpr int kHalfThreads = 32 * (kConverters + 2);
    static constexpr int kHalfWarps = kHalfThreads / 32;
    // Two independent halves per CTA, each with its own warps, shared memory
    // and 256 tensor-memory columns, each working one row block: a CTA that
    // allocates tensor memory gets an SM to itself, and two row blocks in
    // flight let one half's expansion overlap the other's MMAs.
    static constexpr int kThreads = 2 * kHalfThreads;
    static constexpr int kPartN = kN / kSplit;                     // accumulator columns per converter
    static constexpr int kPartUnits = 4 / kSplit;                  // 16-byte code units per group
    static constexpr int kGroupCols = kGemvGroup / 2;              // A columns of one group (bf16x2)
    static constexpr int kACol = 0;                                // A buffers: 2 x 64 columns
    static constexpr int kDCol = 2 * kGroupCols;                   // accumulators: 2 x kN columns
    static constexpr int kTmemCols = 256;
    static constexpr int kBarOff = kXOff + kXStages * kXStageBytes;
    static constexpr int kBars = 2 * kWStages + 2 * kXStages + 4;
    static constexpr int kHalfBytes = (kBarOff + kBars * 8 + 16 + 1023) / 1024 * 1024;
    static constexpr int kSmemBytes = 2 * kHalfBytes + 1024;   // + alignment slack
    static_assert(kN == 32 || kN == 64, "batch columns");
    static_assert(kDCol + 2 * kN <= kTmemCols, "tensor memory");
};

template <int kN>
__global__ void __launch_bounds__(GemvCfg<kN>::kThreads, 1)
int4_gemv_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                 const __grid_constant__ CUtensorMap tmap_s, const GemvArgs a) {
    using C = GemvCfg<kN>;
    constexpr int SW = C::kWStages;
    constexpr int SX = C::kXStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem0 = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int half = warp / C::kHalfWarps;
    const int lwarp = warp - half * C::kHalfWarps;     // warp within the half
    const int rb = 2 * static_cast<int>(blockIdx.x) + half;   // this half's row block
    const bool active = rb < a.n / kGemvRows;
    uint8_t* smem = smem0 + half * C::kHalfBytes;
    uint64_t* full_w = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* empty_w = full_w + SW;
    uint64_t* full_x = empty_w + SW;
    uint64_t* empty_x = full_x + SX;
    uint64_t* a_ready = empty_x + SX;     // [2] A buffer written (the converter warps)
    uint64_t* d_ready = a_ready + 2;      // [2] group's MMAs complete (tcgen05.commit)
    // (shared by both halves: in the first half's region)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem0 + C::kBarOff + C::kBars * 8);
    volatile int* failed = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int row0 = rb * kGemvRows;
    const int KT = a.k / kGemvKTile;
    const int NG = KT * (kGemvKTile / kGemvGroup);    // groups

    launch_dependents();
    if (tid == 0) {
        for (int hf = 0; hf < 2; ++hf) {
            uint64_t* fw = reinterpret_cast<uint64_t*>(smem0 + hf * C::kHalfBytes + C::kBarOff);
            uint64_t* ew = fw + SW;
            uint64_t* fx = ew + SW;
            uint64_t* ex = fx + SX;
            uint64_t* ar = ex + SX;
            uint64_t* dr = ar + 2;
            for (int s = 0; s < SW; ++s) {
                mbar_init(&fw[s], 1);
                mbar_init(&ew[s], C::kConverters);
            }
            for (int s = 0; s < SX; ++s) {
                mbar_init(&fx[s], 1);
                mbar_init(&ex[s], 1);              // the MMA commit
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(&ar[b], C::kConverters);
                mbar_init(&dr[b], 1);
            }
        }
        *failed = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_slot), 2 * C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot + static_cast<uint32_t>(half * C::kTmemCols);   // this half's columns

    if (!active) {
        // (an odd number of row blocks: this half has none)
    } else if (lwarp == C::kConverters) {
        // ================= TMA producers: lane 0 codes, lane 1 x =================
        if (lane == 0) {
            prefetch_tensormap(&tmap_w);
            prefetch_tensormap(&tmap_s);
            // the first code tiles into L2 while the preceding kernel finishes
            const int tile0 = rb * KT;     // first code tile of the row block
            for (int t = 0; t < SW && t < KT; ++t) tma_prefetch_l2_2d(&tmap_w, 0, (tile0 + t) * kGemvRows);
            grid_dependency_wait();
            for (int t = 0; t < KT; ++t) {
                const int stage = t % SW;
                if (t >= SW) gemv_wait(&empty_w[stage], ((t / SW) + 1) & 1, failed, a.status);
                const uint32_t base = smem_addr(smem + stage * C::kWStageBytes);
                mbar_arrive_expect_tx(&full_w[stage], C::kWBytes + C::kSBytes);
                tma_load_2d(base, &tmap_w, 0, (tile0 + t) * kGemvRows, &full_w[stage]);
                tma_load_2d(base + C::kWBytes, &tmap_s, 0,
                            rb * (a.k / kGemvGroup) + t * (kGemvKTile / kGemvGroup), &full_w[stage]);
            }
        } else if (lane == 1) {
            prefetch_tensormap(&tmap_x);
            grid_dependency_wait();
            for (int t = 0; t < KT; ++t) {
                const int stage = t % SX;
                if (t >= SX) gemv_wait(&empty_x[stage], ((t / SX) + 1) & 1, failed, a.status);
                const uint32_t base = smem_addr(smem + C::kXOff + stage * C::kXStageBytes);
                mbar_arrive_expect_tx(&full_x[stage], C::kXStageBytes);
#pragma unroll
                for (int i = 0; i < kGemvKTile / 64; ++i)
                    tma_load_2d(base + i * C::kXBoxBytes, &tmap_x, t * kGemvKTile + i * 64, 0, &full_x[stage]);
            }
        }
    } else if (lwarp == C::kConverters + 1) {
        // ================= MMA issuer =================
        if (lane == 0) {
            constexpr uint32_t idesc = mma_idesc_bf16(kN);
            for (int t = 0; t < KT; ++t) {
                const int stage = t % SX;
                gemv_wait(&full_x[stage], (t / SX) & 1, failed, a.status);
                const uint32_t xaddr = smem_addr(smem + C::kXOff + stage * C::kXStageBytes);
#pragma unroll
                for (int grp = 0; grp < kGemvKTile / kGemvGroup; ++grp) {
                    const int g = t * (kGemvKTile / kGemvGroup) + grp;
                    const int b = g & 1;
                    gemv_wait(&a_ready[b], (g >> 1) & 1, failed, a.status);
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < kGemvGroup / 16; ++j) {
                        // k-step j of the group: x columns 128 grp + 16 j .. +15, in box
                        // (2 grp + j / 4) at byte 32 (j mod 4) of each 128-byte row
                        const uint32_t xk = xaddr + (2 * grp + j / 4) * C::kXBoxBytes + 32 * (j % 4);
                        tc_mma_ts(tmem + C::kDCol + b * kN, tmem + C::kACol + b * C::kGroupCols + 8 * j,
                                  sw128_kmajor_desc(xk), idesc, j > 0 ? 1u : 0u);
                    }
                    tc_commit(&d_ready[b]);
                }
                tc_commit(&empty_x[stage]);    // this stage's x reads are done
            }
        }
    } else {
        // ====== converters: warp w owns rows 32 (w mod 4) .., part w / 4 ======
        // (thread = row = tensor-memory lane; the part picks 1 / kSplit of a
        // group's columns for A and of the batch columns for the output)
        constexpr int PU = C::kPartUnits;
        // (a warp reaches the tensor-memory lanes 32 (w mod 4) .. of its
        // index w in the CTA)
        const int quarter = warp & 3;
        const int part = lwarp >> 2;
        const int r = 32 * quarter + lane;                         // row in the tile
        const uint32_t tlane = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
        float acc[C::kPartN];
#pragma unroll
        for (int n = 0; n < C::kPartN; ++n) acc[n] = 0.f;
        float s_cur[2] = {0.f, 0.f}, s_prev[2] = {0.f, 0.f};

        // acc += s * (this row's part of the accumulator of group g)
        auto readout = [&](int g, float s) {
            const int b = g & 1;
            gemv_wait(&d_ready[b], (g >> 1) & 1, failed, a.status);
            tc_fence_after();
            const uint32_t dcol = tlane + C::kDCol + b * kN + part * C::kPartN;
#pragma unroll
            for (int q = 0; q < C::kPartN / 16; ++q) {
                uint32_t v[16];
                tmem_ld16(dcol + 16 * q, v);
                tmem_wait_ld(v);
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[16 * q + i] = fmaf(s, __uint_as_float(v[i]), acc[16 * q + i]);
            }
        };

        for (int t = 0; t < KT; ++t) {
            const int stage = t % SW;
            gemv_wait(&full_w[stage], (t / SW) & 1, failed, a.status);
            const uint32_t wrow = smem_addr(smem + stage * C::kWStageBytes) + r * 128;
            const uint16_t* sb = reinterpret_cast<const uint16_t*>(smem + stage * C::kWStageBytes + C::kWBytes);
            // this row's code units of this part: group grp, units 4 grp + PU part + e;
            // 16-byte unit u of a row sits at unit u ^ (r mod 8)
            uint4 raw[2 * PU];
#pragma unroll
            for (int grp = 0; grp < 2; ++grp)
#pragma unroll
                for (int e = 0; e < PU; ++e) {
                    const int u = 4 * grp + PU * part + e;
                    raw[PU * grp + e] = lds128(wrow + ((u ^ (r & 7)) << 4));
                }
            s_prev[0] = s_cur[0];
            s_prev[1] = s_cur[1];
            s_cur[0] = bf16_bits_to_f32(sb[r]);
            s_cur[1] = bf16_bits_to_f32(sb[kGemvRows + r]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_w[stage]);     // codes and scales are in registers

#pragma unroll
            for (int grp = 0; grp < kGemvKTile / kGemvGroup; ++grp) {
                const int g = t * (kGemvKTile / kGemvGroup) + grp;
                const int b = g & 1;
                // group g - 2 used the same A and accumulator buffers: read its
                // result out (its MMAs are then complete) before overwriting A
                if (g >= 2) readout(g - 2, s_prev[grp]);
                // expand this part of the group's codes: unit e gives 16 bf16x2 A
                // columns, column 4w + i = columns (8w + 2i, 8w + 2i + 1) of the unit
#pragma unroll
                for (int e = 0; e < PU; ++e) {
                    const uint32_t wds[4] = {raw[PU * grp + e].x, raw[PU * grp + e].y, raw[PU * grp + e].z,
                                             raw[PU * grp + e].w};
                    uint32_t v[16];
#pragma unroll
                    for (int w = 0; w < 4; ++w)
#pragma unroll
                        for (int i = 0; i < 4; ++i) v[4 * w + i] = int4_pair_to_bf16x2(wds[w] >> (4 * i));
                    tmem_st16(tlane + C::kACol + b * C::kGroupCols + 16 * (PU * part + e), v);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a_ready[b]);
            }
        }
        // the last two groups
        for (int g = (NG >= 2 ? NG - 2 : 0); g < NG; ++g) readout(g, s_cur[g & 1]);

        grid_dependency_wait();
#pragma unroll
        for (int n = 0; n < C::kPartN; ++n) {
            const int bn = part * C::kPartN + n;
            if (bn < a.batch) a.y[static_cast<int64_t>(bn) * a.n + row0 + r] = f32_to_bf16_bits(acc[n]);
        }
    }

    // every tensor-memory access and MMA of this CTA is complete here (the
    // converters waited for the last groups' commits): free the columns
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(*tmem_slot, 2 * C::kTmemCols);
    }
}

int gemv_batch_cols(int batch) { return batch <= 32 ? 32 : 64; }

#define PKV_GEMV_DISPATCH(ncols, EXPR) \
    switch (ncols) {                     \
        case 32: { constexpr int N = 32; EXPR; } \
        case 64: { constexpr int N = 64; EXPR; } \
        default: return cudaErrorInvalidValue; \
    }

cudaError_t gemv_set_smem_attr(int ncols) {
    PKV_GEMV_DISPATCH(ncols, return cudaFuncSetAttribute(int4_gemv_kernel<N>,
                                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                         GemvCfg<N>::kSmemBytes))
}

cudaError_t launch_int4_gemv(int ncols, cudaStream_t stream, const CUtensorMap& tmap_w,
                             const CUtensorMap& tmap_x, const CUtensorMap& tmap_s, const GemvArgs& args) {
    PKV_GEMV_DISPATCH(ncols, {
        PdlLaunch l(dim3((args.n / kGemvRows + 1) / 2), dim3(GemvCfg<N>::kThreads), GemvCfg<N>::kSmemBytes,
                    stream);
        return cudaLaunchKernelEx(&l.cfg, int4_gemv_kernel<N>, tmap_w, tmap_x, tmap_s, args);
    })
}

}  // namespace pkv
