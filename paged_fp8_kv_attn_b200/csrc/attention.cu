// attention.cu -- paged decode attention over an FP8 E4M3 or BF16 KV cache
// for sm_100a: split-K partial kernel plus log-sum-exp merge kernel.
//
// Source pages: "大模型推理优化：量化、压缩与安全验证", section "量化 KV cache"
// (FP8 e4m3 cache; the FP8 attention kernel converts values on every read);
// siami.tw editorial, section "KV 快取量化" (Table 1: FP8 vs BF16 KV decode
// throughput); remio.ai commentary, section "小型缓存胜过单纯的速度" (decode
// is memory-bound).  The pages give no kernel design; the one here is:
//
//  * Work: units are (request, KV head, 64-token chunk).  The units of the
//    whole batch are cut into num_ctas equal contiguous ranges, one per CTA
//    of a single persistent wave, so long and short requests balance.  A CTA
//    walks its range as "segments" (maximal runs inside one (request, KV
//    head) item).  A segment covering a whole item writes the final output;
//    otherwise it writes an fp32 partial (m, l, O) to workspace slot
//    cta + item (unique because the partition is monotone) and the merge
//    kernel combines the partials of that item.
//  * Pipeline: warp 4 is the producer.  Its lane 0 streams the K and V tiles
//    of each chunk from the [page][kv_head][slot][dim] pools into a ring of
//    shared-memory stages with 2-D TMA tensor loads (128-byte swizzle)
//    completing on mbarriers; consumers release a stage through a second
//    mbarrier.  Before its grid-dependency wait the producer prefetches its
//    first stages into L2 so the preceding kernels (tag check, append)
//    overlap with DRAM traffic.
//  * Math: warps 0-3 each own a 16-token slice of every chunk and keep their
//    own online-softmax state.  Scores S = Q K^T and the output O = P V run on
//    tensor cores as m16n8k16 MMAs with the query heads of one KV head (the
//    GQA group, padded to 8 or 16) as the M dimension.  FP8 codes are turned
//    into f16 in registers with the hardware E4M3 conversion (exact); the
//    per-tensor scales are folded into the score scale and into the output.
//    For the FP8 path each query head is scaled by a power of two so that
//    its largest |q| lies in [128, 256), which keeps the bf16 -> f16
//    conversion exact; the power of two is undone in the score scale.
//  * Layout tricks: the token order inside each 8-row group and the order of
//    the head dimension inside the QK contraction are permuted (both are
//    free: softmax and the contraction are invariant under them) so that
//    each thread's shared-memory reads are 16-byte (K) or 4-byte (V) words
//    that hit 32 distinct banks under the TMA swizzle.
//  * Lazy rescaling: a warp rescales O only when a head's running maximum
//    grows by more than 8 (log2 units); P is then at most 2^8, exact enough
//    in f16 and far from overflow.
#include "device.cuh"
#include "internal.h"

namespace pkv {

constexpr int kConsumerWarps = 4;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;
constexpr float kNegInf = -__builtin_huge_valf();

template <bool kFp8, int kD, int kGP, int kH>
struct AttnCfg {
    static constexpr int kElem = kFp8 ? 1 : 2;
    static constexpr int kRowBytes = kD * kElem;                 // 64, 128 or 256
    static constexpr int kBoxBytes = kFp8 ? kRowBytes : 128;     // TMA box inner bytes
    static constexpr int kSubTiles = kRowBytes / kBoxBytes;      // 2 for BF16 D=128
    static constexpr int kSwizzle = kBoxBytes;                   // 128 or 64
    static constexpr int kSubTileBytes = kChunkTokens * kBoxBytes;
    static constexpr int kHeadTileBytes = kChunkTokens * kRowBytes;  // one KV head of a chunk
    static constexpr int kTileBytes = kH * kHeadTileBytes;           // K (or V) of a stage
    static constexpr int kStageBytes = 2 * kTileBytes;
    // Pipeline depth and resident CTAs per SM, chosen by measurement on B200:
    // resident warps matter more than depth (each CTA keeps up to kStages
    // chunks in flight), so the depth is the largest that still lets
    // kMinBlocks CTAs share an SM's 228 KB of shared memory.
    static constexpr int kStages = kFp8 ? (kD == 128 ? (kH == 2 ? 3 : 4) : (kH == 2 ? 3 : 6))
                                        : (kD == 128 ? 2 : 4);
    static constexpr int kMinBlocks = (kFp8 && kGP == 8 && kH == 1) ? 3 : 2;
    // The epilogue's cross-warp reduction of O (4 warps x kGP heads x kD fp32)
    // reuses the stage of the segment's last chunk when it fits there (a
    // group of 8: exactly one FP8 stage), which is released to the producer
    // only after the epilogue; otherwise it has its own buffer.
    static constexpr bool kRedInStage = kConsumerWarps * kGP * kD * 4 <= kStageBytes;
    static constexpr int kRedOff = kStages * kStageBytes;
    static constexpr int kRedFloats = kConsumerWarps * kGP * ((kRedInStage ? 0 : kD) + 3);
    static constexpr int kBarOff = kRedOff + kRedFloats * 4;
    static constexpr int kFlagOff = kBarOff + 2 * kStages * 8;
    static constexpr int kScratchOff = kFlagOff + kStages * 4;
    // Cluster mode: the partial result of one item (O[kRecHeads][kD], then
    // (m, l, lr, 0) per head, fp32) kept in shared memory for the cluster's
    // reduction.  A CTA's first segment uses the dedicated buffer at kRecOff;
    // its last one a pipeline stage (all free by then).  The cluster table
    // holds, per (rank, record), the item and the record's address.
    static constexpr int kRecHeads = kH * kGP;
    static constexpr int kRecBytes = kRecHeads * kD * 4 + 4 * kRecHeads * 4;
    static constexpr int kCluOff = kScratchOff + 16 * 4;
    static constexpr int kCluInts = 4 * kMaxCluster + 2 * kMaxCluster * kMaxCluster + 1;
    static constexpr int kRecOff = (kCluOff + kCluInts * 4 + 15) / 16 * 16;
    static constexpr int kSmemBytes = kRecOff + kRecBytes + 1024;  // + alignment slack
    static_assert(kRecBytes <= kStageBytes, "a record must fit in one stage");
    // Registers per thread holding a segment's raw query words.  They are
    // loaded before the previous segment's epilogue when that adds at most
    // 16 live registers to a variant with the 2-CTA register budget (168);
    // otherwise (more words, or the tighter 3-CTA budget) at the segment's
    // start.
    static constexpr int kQWords = kFp8 ? (kGP / 8) * (kD / 64) * 8 : (kGP / 8) * (kD / 16) * 2;
    static constexpr bool kEarlyQ = kQWords <= 16 && kMinBlocks == 2;
    static_assert(kD == 64 || kD == 128, "head_dim");
    static_assert(kGP == 8 || kGP == 16, "group pad");
    static_assert(kH == 1 || (kH == 2 && kGP == 8), "two KV heads per item need a group <= 8");
};

// XOR applied to the 16-byte unit index of the epilogue's O rows written by
// lanes with thread-in-group c (rows 2c, 2c+1 of each 8-head block).  Chosen
// per accumulator layout so that one store instruction's lanes (and each
// 8-lane phase of a 16-byte store) reach distinct banks: FP8 D=128 stores
// units 4g+k, FP8 D=64 units 2g+k, BF16 single words of units 4mb+g/4 (+2).
template <bool kFp8, int kD>
__device__ __forceinline__ uint32_t red_swizzle(int c) {
    if constexpr (!kFp8) return 2u * c;
    else if constexpr (kD == 128) return static_cast<uint32_t>(c);
    else return static_cast<uint32_t>((c & 1) | ((c & 2) << 1));
}

// Token permutation inside an 8-row group: row tau(n) feeds MMA column n.
__device__ __forceinline__ int tau(int n) { return n ^ ((n & 1) << 2); }

struct Segment {
    int b, h, c0, c1, n, L;
};

// Walks a CTA's unit range [u, u_hi) segment by segment.  Every warp runs an
// identical copy, so producer and consumers agree without communicating.
// Units of an item are its chunks from the request's first chunk (0, or
// chunk_begin[b] in shared-prefix mode) to its last.
struct Walker {
    const int32_t* seq_lens;
    const int32_t* chunk_begin;   // null: every request from chunk 0
    int64_t max_tokens;
    int num_kv_heads;
    int batch;
    int b, h, ch, n, L, cb;
    int64_t u, u_hi;

    __device__ __forceinline__ int chunks_of(int32_t len) const {
        return (len >= 1 && static_cast<int64_t>(len) <= max_tokens)
                   ? (len + kChunkTokens - 1) / kChunkTokens
                   : 0;
    }
    __device__ __forceinline__ int begin_of(int bb) const {
        return chunk_begin != nullptr ? chunk_begin[bb] : 0;
    }
    // units of one item of request bb
    __device__ __forceinline__ int units_of(int bb, int32_t len) const {
        const int c = chunks_of(len);
        return c > 0 ? c - begin_of(bb) : 0;
    }
    __device__ __forceinline__ void init(int b0, int pre0, int64_t ulo, int64_t uhi) {
        u = ulo;
        u_hi = uhi;
        b = b0;
        h = ch = n = L = cb = 0;
        if (u < u_hi) {
            L = seq_lens[b];
            n = chunks_of(L);
            cb = begin_of(b);
            const int64_t off = ulo - static_cast<int64_t>(num_kv_heads) * pre0;
            h = static_cast<int>(off / (n - cb));
            ch = cb + static_cast<int>(off % (n - cb));
        }
    }
    __device__ __forceinline__ bool next(Segment& s) {
        if (u >= u_hi || ch >= n) {   // ch >= n only if the batch changed under us
            u = u_hi;
            return false;
        }
        const int64_t left = u_hi - u;
        const int take = static_cast<int>(left < (n - ch) ? left : (n - ch));
        s.b = b;
        s.h = h;
        s.c0 = ch;
        s.c1 = ch + take;
        s.n = n;
        s.L = L;
        u += take;
        ch += take;
        if (u < u_hi && ch == n) {
            if (++h == num_kv_heads) {
                h = 0;
                // (requests with no units: invalid lengths, and in shared-prefix
                // mode requests the shared pass finishes)
                do {
                    ++b;
                    L = seq_lens[b];
                    n = chunks_of(L);
                    cb = begin_of(b);
                } while ((n == 0 || cb >= n) && b + 1 < batch);
            }
            ch = cb;
        }
        return true;
    }
};

// Bounded mbarrier wait.  After a timeout in this CTA every later wait
// returns at once, so the kernel always runs to completion; the workspace
// status word (cleared by CTA 0 when the kernel starts) reports the failure.
__device__ __forceinline__ void wait_or_give_up(uint64_t* bar, uint32_t parity,
                                                volatile int* cta_failed, uint32_t* status) {
    if (mbar_try_wait(bar, parity)) return;   // the common case: already complete
    if (*cta_failed) return;
    if (!mbar_wait(bar, parity)) {
        *cta_failed = 1;
        atomicOr(status, 1u);
    }
}

// Page id of entry j of a row, read through a 32-entry window held across
// the producer warp's lanes (one coalesced load per 32 pages).
struct PageWindow {
    const int32_t* row;
    int base;
    int32_t mine;
    __device__ __forceinline__ void reset(const int32_t* r) {
        row = r;
        base = -(1 << 30);
    }
    // Issues the load of the window starting at entry j ahead of its use.
    __device__ __forceinline__ void preload(int j, int limit, int lane) {
        base = j;
        mine = (j + lane < limit) ? row[j + lane] : -1;
    }
    __device__ __forceinline__ int32_t get(int j, int limit, int lane) {
        if (j < base || j >= base + 32) {
            base = j;
            mine = (j + lane < limit) ? row[j + lane] : -1;
        }
        return __shfl_sync(0xffffffffu, mine, j - base);
    }
};

// ---------------------------------------------------------------------------
// cluster mode: combine the split items inside the cluster
// ---------------------------------------------------------------------------
// Every CTA of the cluster, all threads, after its walk.  The records of one
// item sit in consecutive ranks (the ranges are contiguous and increasing), so
// in (rank, record) order each split item's records form one run; the runs'
// outputs are spread over all threads of the cluster.  Kept out of line so
// that nothing it needs stays live through the partial kernel's main loop.
template <bool kFp8, int kD, int kGP, int kH>
__device__ __noinline__ void attn_cluster_reduce(const AttnArgs& a, uint8_t* smem) {
    using C = AttnCfg<kFp8, kD, kGP, kH>;
    constexpr int K = kMaxCluster;
    constexpr int kWarps = kAttnThreads / 32;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    int* const scratch = reinterpret_cast<int*>(smem + C::kScratchOff);
    float* const rec0 = reinterpret_cast<float*>(smem + C::kRecOff);
    // per split item: its id, its records' cluster-window addresses (at most
    // one per rank and record slot) and their count
    int* const s_item = reinterpret_cast<int*>(smem + C::kCluOff);        // [2K]
    int* const s_count = s_item + 2 * K;                                    // [2K]
    uint32_t* const s_list = reinterpret_cast<uint32_t*>(s_count + 2 * K);  // [2K][K]
    int* const n_split = reinterpret_cast<int*>(s_list + 2 * K * K);
    // the arguments used below, in registers
    const int B = a.batch, IPR = a.items_per_req, CS = a.cluster_size, NCL = a.num_clusters;
    const int IQ = kH * a.group, Hq = a.num_q_heads;
    const int32_t* const seq_lens = a.seq_lens;
    uint16_t* const out = a.out;
    float* const lse = a.lse;
    const int64_t max_tokens = static_cast<int64_t>(a.max_pages) * a.page_size;
    const int crank = static_cast<int>(blockIdx.x % CS);

    // Requests with no chunks (invalid length) among the cluster's items
    // produce no record: rank 0 writes their dead outputs, one warp per item,
    // while the other CTAs of the cluster are still arriving.
    if (crank == 0) {
        const int cid = static_cast<int>(blockIdx.x) / CS, I = B * IPR;
        const int i0 = static_cast<int>(static_cast<int64_t>(cid) * I / NCL);
        const int i1 = static_cast<int>(static_cast<int64_t>(cid + 1) * I / NCL);
        for (int item = i0 + warp; item < i1; item += kWarps) {
            const int b = item / IPR, h = item - b * IPR;
            const int32_t len = seq_lens[b];
            if (len >= 1 && static_cast<int64_t>(len) <= max_tokens) continue;
            const int64_t row0 = static_cast<int64_t>(b) * Hq + static_cast<int64_t>(h) * IQ;
            for (int e = lane; e < IQ * kD; e += 32) out[row0 * kD + e] = 0;
            if (lane < IQ) lse[row0 + lane] = kNegInf;
        }
    }

    cluster_sync_all();   // every record of the cluster is written
    if (warp == 0) {
        // Lane e < 2 CS reads record e (rank e / 2, slot e % 2): its item and,
        // for slot 1, the address of the rank's stage-resident record.  In
        // this order the records of one item are consecutive (empty records
        // aside), so the split items and their record lists follow from masks.
        int item = -1;
        uint32_t addr = 0;
        if (lane < 2 * CS) {
            const uint32_t r = static_cast<uint32_t>(lane >> 1), slot = static_cast<uint32_t>(lane & 1);
            item = ld_cluster_s32(cluster_map(smem_addr(&scratch[5 + slot]), r));
            const uint32_t rec1 =
                static_cast<uint32_t>(ld_cluster_s32(cluster_map(smem_addr(&scratch[7]), r)));
            addr = cluster_map(slot == 0 ? smem_addr(rec0) : rec1, r);
        }
        const uint32_t valid = __ballot_sync(0xffffffffu, item >= 0);
        const uint32_t below = (1u << lane) - 1u;
        // the nearest valid record before this one, and its item
        const uint32_t vb = valid & below;
        const int prev_lane = vb ? 31 - __clz(vb) : 0;
        const int prev_item = __shfl_sync(0xffffffffu, item, prev_lane);
        const bool starts = item >= 0 && (vb == 0 || prev_item != item);
        const uint32_t starts_mask = __ballot_sync(0xffffffffu, starts);
        if (item >= 0) {
            const uint32_t sb = starts_mask & (below | (1u << lane));
            const int first = 31 - __clz(sb);                  // this item's first record
            const int j = __popc(sb) - 1;                      // its split-item index
            const int k = __popc(valid & below & ~((1u << first) - 1u));   // position in its list
            s_list[j * K + k] = addr;
            if (starts) {
                const uint32_t later = starts_mask & ~(below | (1u << lane));
                const int next = later ? __ffs(later) - 1 : 32;
                const uint32_t span = (next == 32 ? 0xffffffffu : ((1u << next) - 1u)) & ~below;
                s_item[j] = item;
                s_count[j] = __popc(valid & span);
            }
        }
        if (lane == 0) *n_split = __popc(starts_mask);
    }
    __syncthreads();

    // One warp per (split item, query head), spread over the cluster's ranks:
    // lane k < n loads record k's (m, l, lr) (one round trip), the weights are
    // shared by shuffles, then lane q sums output quad q over the n records
    // with all n loads in flight (a second round trip).
    constexpr uint32_t kMlOff = C::kRecHeads * kD * 4;   // byte offset of (m, l, lr, 0) per head
    constexpr int kQuads = kD / 4;                       // 32 (D = 128) or 16 (D = 64)
    const int pairs = *n_split * IQ;
    for (int pr = crank + CS * warp; pr < pairs; pr += CS * kWarps) {
        const int j = pr / IQ, hq = pr - j * IQ;
        const int n = s_count[j];
        const uint32_t* const list = s_list + j * K;
        float4 ml = make_float4(kNegInf, 0.f, 0.f, 0.f);
        if (lane < n) ml = ld_cluster_f32x4(list[lane] + kMlOff + 16 * hq);
        float M = ml.x;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        const float wt = (lane < n && ml.x != kNegInf) ? exp2f(ml.x - M) : 0.f;
        float Lsum = wt * ml.y, Lr = wt * ml.z;
        int dead = lane < n && ml.y < 0.f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            Lsum += __shfl_xor_sync(0xffffffffu, Lsum, off);
            Lr += __shfl_xor_sync(0xffffffffu, Lr, off);
        }
        dead = __any_sync(0xffffffffu, dead);
        const int item = s_item[j];
        const int b = item / IPR, h = item - b * IPR;
        const int64_t hrow = static_cast<int64_t>(b) * Hq + static_cast<int64_t>(h) * IQ + hq;
        if (lane < kQuads) {
            float4 x[K];
#pragma unroll
            for (int k = 0; k < K; ++k)
                if (k < n) x[k] = ld_cluster_f32x4(list[k] + (hq * kD + 4 * lane) * 4);
            float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int k = 0; k < K; ++k) {
                const float w = __shfl_sync(0xffffffffu >> (32 - kQuads), wt, k);
                if (k < n) {
                    O.x += w * x[k].x;
                    O.y += w * x[k].y;
                    O.z += w * x[k].z;
                    O.w += w * x[k].w;
                }
            }
            uint32_t* dst = reinterpret_cast<uint32_t*>(out + hrow * kD + 4 * lane);
            if (dead) {
                dst[0] = 0u;
                dst[1] = 0u;
            } else {
                dst[0] = pack_bf16x2(O.x / Lr, O.y / Lr);
                dst[1] = pack_bf16x2(O.z / Lr, O.w / Lr);
            }
        }
        if (lane == 0) lse[hrow] = dead ? kNegInf : (M + log2f(Lsum)) * kLn2;
    }
    cluster_sync_all();   // no CTA leaves while another may read its records
}

// ---------------------------------------------------------------------------
// the split-K partial kernel
// ---------------------------------------------------------------------------
template <bool kFp8, int kD, int kGP, int kH>
__global__ void __launch_bounds__(kAttnThreads, (AttnCfg<kFp8, kD, kGP, kH>::kMinBlocks))
attn_partial_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ AttnArgs a) {
    using C = AttnCfg<kFp8, kD, kGP, kH>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float* red_m = reinterpret_cast<float*>(smem + C::kRedOff);
    float* red_l = red_m + kConsumerWarps * kGP;
    float* red_lr = red_l + kConsumerWarps * kGP;
    float* const red_o_own = red_lr + kConsumerWarps * kGP;   // used when !kRedInStage
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* empty_bar = full_bar + S;
    volatile int* stage_bad = reinterpret_cast<volatile int*>(smem + C::kFlagOff);
    // read after the stage's full barrier, whose wait orders it after the write
    const int* stage_bad_rd = reinterpret_cast<const int*>(smem + C::kFlagOff);
    int* scratch = reinterpret_cast<int*>(smem + C::kScratchOff);
    volatile int* cta_failed = scratch + 10;
    // cluster mode: scratch[5], scratch[6] = item of this CTA's first / last
    // partial record (-1: none); scratch[7] = shared address of the last one
    float* const rec0 = reinterpret_cast<float*>(smem + C::kRecOff);
    const bool clu = a.cluster_size > 0;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int B = a.batch;
    const int Hkv = a.num_kv_heads;        // KV heads of the pool
    const int IPR = a.items_per_req;       // work items per request (Hkv / kH)
    const int64_t max_tokens = static_cast<int64_t>(a.max_pages) * a.page_size;

    launch_dependents();
    // Shared-prefix mode: the chunk begins the partition needs come from the
    // plan kernels that precede this one.
    if (a.chunk_begin != nullptr) grid_dependency_wait();
    // The call's status word starts at zero.  Clearing it before the grid
    // dependency wait is safe: no kernel reads it (the caller reads it in
    // stream order, after the call), and a bounded wait of this call can only
    // expire seconds after CTA 0, the first to be scheduled, has run this.
    // (in shared-prefix mode the plan kernel that opens the call clears it)
    if (blockIdx.x == 0 && tid == 0 && a.chunk_begin == nullptr) *a.ws_status = 0u;
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kConsumerWarps);
        }
        *cta_failed = 0;
        scratch[5] = -1;
        scratch[6] = -1;
        scratch[7] = 0;
        fence_barrier_init();
    }

    // ---- partition: exclusive scan of chunk counts over the batch --------
    Walker walk;
    walk.seq_lens = a.seq_lens;
    walk.chunk_begin = a.chunk_begin;
    walk.max_tokens = max_tokens;
    walk.num_kv_heads = IPR;
    walk.batch = B;
    const int per = (B + kAttnThreads - 1) / kAttnThreads;
    const int b_lo = min(B, tid * per);
    const int b_hi = min(B, b_lo + per);
    int local = 0;
    for (int b = b_lo; b < b_hi; ++b) local += walk.units_of(b, a.seq_lens[b]);
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    int warp_base = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kAttnThreads / 32; ++w) {
        const int t = scratch[w];
        if (w < warp) warp_base += t;
        total += t;
    }
    const int64_t U = static_cast<int64_t>(IPR) * total;
    const int run0 = warp_base + incl - local;   // chunks of the requests before b_lo
    int64_t u_lo, u_hi;
    if (!clu) {
        // The units are cut over NE = min(grid, U) CTAs, so that every CTA of
        // the partition holds at least one unit and therefore writes the
        // partial of every item it touches: the merge reads only slots written
        // by this call (the rest of the grid, if any, has nothing to do).
        const int64_t NE = U < a.num_ctas ? U : a.num_ctas;
        u_lo = (blockIdx.x < NE) ? static_cast<int64_t>(blockIdx.x) * U / NE : U;
        u_hi = (blockIdx.x < NE) ? static_cast<int64_t>(blockIdx.x + 1) * U / NE : U;
    } else {
        // Cluster mode: cluster k owns the items [k I / K, (k+1) I / K) (I
        // items, K clusters), so no item crosses a cluster; its units are cut
        // evenly over the cluster's CTAs.  Unit offset of item i = b IPR + h:
        // IPR * (chunks of the requests before b) + h * (chunks of b).
        const int CS = a.cluster_size;
        const int cid = blockIdx.x / CS;
        const int crank = blockIdx.x % CS;
        const int I = B * IPR;
        const int i0 = static_cast<int>(static_cast<int64_t>(cid) * I / a.num_clusters);
        const int i1 = static_cast<int>(static_cast<int64_t>(cid + 1) * I / a.num_clusters);
        int run = run0;
        for (int b = b_lo; b < b_hi; ++b) {
            const int n = walk.units_of(b, a.seq_lens[b]);
            if (b == i0 / IPR) { scratch[11] = run; scratch[12] = n; }
            if (b == i1 / IPR) { scratch[13] = run; scratch[14] = n; }
            run += n;
        }
        __syncthreads();
        const int64_t c_lo = (i0 >= I) ? U : static_cast<int64_t>(IPR) * scratch[11] +
                                                 static_cast<int64_t>(i0 % IPR) * scratch[12];
        const int64_t c_hi = (i1 >= I) ? U : static_cast<int64_t>(IPR) * scratch[13] +
                                                 static_cast<int64_t>(i1 % IPR) * scratch[14];
        u_lo = c_lo + static_cast<int64_t>(crank) * (c_hi - c_lo) / CS;
        u_hi = c_lo + static_cast<int64_t>(crank + 1) * (c_hi - c_lo) / CS;
    }
    {
        int run = run0;
        for (int b = b_lo; b < b_hi; ++b) {
            const int n = walk.units_of(b, a.seq_lens[b]);
            if (n > 0 && u_lo < u_hi && static_cast<int64_t>(IPR) * run <= u_lo &&
                u_lo < static_cast<int64_t>(IPR) * (run + n)) {
                scratch[8] = b;
                scratch[9] = run;
            }
            run += n;
        }
    }
    __syncthreads();
    if (u_lo >= u_hi && !clu) return;   // nothing to do (the merge reads no slot of this CTA)
    // (an empty range in cluster mode: the walk yields nothing and the CTA
    // only takes part in its cluster's reduction)
    walk.init(u_lo < u_hi ? scratch[8] : 0, u_lo < u_hi ? scratch[9] : 0, u_lo, u_hi);


    const int P = a.page_size;
    const int box_rows = a.box_rows;
    // With two KV heads per item and 64-token pages, the item's K (or V) rows
    // of a page are one contiguous 128-row box; otherwise one box per KV head
    // and page (per 64 rows for 128-token pages).
    const bool joint = (kH == 2) && (box_rows == 2 * kChunkTokens);
    const int boxes = joint ? 1 : kChunkTokens / box_rows;

    if (warp == kConsumerWarps) {
        // ================= producer warp =================
        prefetch_tensormap(&tmap_k);
        prefetch_tensormap(&tmap_v);
        PageWindow win;
        win.reset(nullptr);
        // L2 prefetch of the first S chunks, before the dependency wait.
        {
            Walker w2 = walk;
            Segment s;
            int count = 0;
            while (count < S && w2.next(s)) {
                win.reset(a.page_table + static_cast<int64_t>(s.b) * a.max_pages);
                const int npages = (s.L + P - 1) / P;
                for (int ch = s.c0; ch < s.c1 && count < S; ++ch, ++count) {
                    for (int i = 0; i < boxes; ++i) {
                        const int tok0 = ch * kChunkTokens + i * box_rows;
                        const int j = tok0 / P;
                        if (j >= npages) break;
                        const int32_t pid = win.get(j, npages, lane);
                        if (lane == 0 && pid >= 0 && pid < a.num_pages) {
                            for (int kv = 0; kv < (joint ? 1 : kH); ++kv) {
                                const int32_t y = (pid * Hkv + s.h * kH + kv) * P + (tok0 % P);
                                for (int st = 0; st < C::kSubTiles; ++st) {
                                    tma_prefetch_l2_2d(&tmap_k, st * 64, y);
                                    tma_prefetch_l2_2d(&tmap_v, st * 64, y);
                                }
                            }
                        }
                    }
                }
            }
        }
        grid_dependency_wait();
        // A segment's abort flag and first page-table window are loaded one
        // segment ahead, so the first TMA of a segment waits on no load.
        // (the page table is not written by the preceding kernels, so a window
        // the L2 prefetch above already loaded for this row is kept)
        auto load_meta = [&](const Segment& sg, PageWindow& w) {
            const int32_t* row = a.page_table + static_cast<int64_t>(sg.b) * a.max_pages;
            const int j0 = sg.c0 * kChunkTokens / P;
            if (w.row != row || w.base != j0) {
                w.reset(row);
                w.preload(j0, (sg.L + P - 1) / P, lane);
            }
            return (a.abort != nullptr) ? static_cast<int>(a.abort[sg.b]) : 0;
        };
        uint32_t it = 0;
        Segment s;
        bool have = walk.next(s);
        int aborted = have ? load_meta(s, win) : 0;
        while (have) {
            Segment sn;
            const bool have_next = walk.next(sn);
            PageWindow next_win;
            const int next_aborted = have_next ? load_meta(sn, next_win) : 0;
            if (aborted) {
                win = next_win;
                aborted = next_aborted;
                s = sn;
                have = have_next;
                continue;
            }
            // the consumers load this segment's query rows at the end of the
            // previous one: start bringing them into L2 now
            {
                const int64_t q0 = (static_cast<int64_t>(s.b) * a.num_q_heads +
                                    static_cast<int64_t>(s.h) * kH * a.group) * kD;
                if (lane * 64 < kH * a.group * kD) prefetch_l2(a.q + q0 + lane * 64);
            }
            const int npages = (s.L + P - 1) / P;
            for (int ch = s.c0; ch < s.c1; ++ch, ++it) {
                const int stage = it % S;
                if (it >= static_cast<uint32_t>(S)) {
                    if (lane == 0) wait_or_give_up(&empty_bar[stage], ((it / S) + 1) & 1, cta_failed, a.ws_status);
                    __syncwarp();
                }
                const uint32_t kdst = smem_addr(smem + stage * C::kStageBytes);
                const uint32_t vdst = kdst + C::kTileBytes;
                uint32_t bytes = 0;
                int bad = 0;
                int32_t pids[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    pids[i] = -1;
                    if (i < boxes) {
                        const int tok0 = ch * kChunkTokens + i * box_rows;
                        const int j = tok0 / P;
                        if (j < npages) {
                            pids[i] = win.get(j, npages, lane);
                            if (pids[i] < 0 || pids[i] >= a.num_pages) {
                                bad = 1;
                                pids[i] = -1;
                            } else {
                                bytes += 2u * C::kSubTiles * box_rows * C::kBoxBytes * (joint ? 1 : kH);
                            }
                        }
                    }
                }
                if (lane == 0) {
                    stage_bad[stage] = bad;
                    mbar_arrive_expect_tx(&full_bar[stage], bytes);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (pids[i] < 0) continue;
                        const int tok0 = ch * kChunkTokens + i * box_rows;
                        for (int kv = 0; kv < (joint ? 1 : kH); ++kv) {
                            const int32_t y = (pids[i] * Hkv + s.h * kH + kv) * P + (tok0 % P);
                            for (int st = 0; st < C::kSubTiles; ++st) {
                                const uint32_t off = kv * C::kHeadTileBytes + st * C::kSubTileBytes +
                                                     i * box_rows * C::kBoxBytes;
                                tma_load_2d(kdst + off, &tmap_k, st * 64, y, &full_bar[stage]);
                                tma_load_2d(vdst + off, &tmap_v, st * 64, y, &full_bar[stage]);
                            }
                        }
                    }
                }
                __syncwarp();
            }
            win = next_win;
            aborted = next_aborted;
            s = sn;
            have = have_next;
        }
        if (a.cluster_size > 0) attn_cluster_reduce<kFp8, kD, kGP, kH>(a, smem);
        return;
    }

    // ================= consumer warps =================
    // Per warp and chunk: the 16 token rows rb..rb+15.  S = K Q^T and
    // O^T = V^T P^T run as m16n8k16 MMAs whose M dimension is 16 tokens (QK)
    // or 16 head dimensions (PV) and whose N dimension is 8 query heads of
    // the GQA group (kNB n-blocks of 8).  P is moved from the S accumulator
    // layout into the PV B-operand layout with an in-register 8x8 transpose.
    grid_dependency_wait();
    const int g = lane >> 2;   // MMA group id
    const int c = lane & 3;    // thread in group
    const int G = a.group;
    const int IQ = kH * G;                 // query heads of one item
    // Warp -> (KV head of the item, rows of each chunk): with one KV head per
    // item each warp owns 16 rows; with two, two warps share a head and each
    // owns 32 rows (two 16-row MMA tiles).
    constexpr int kWarpsPerHead = kConsumerWarps / kH;
    const int kvh_w = warp / kWarpsPerHead;
    const int row0 = (warp % kWarpsPerHead) * 16 * kH;
    constexpr int kNB = kGP / 8;      // n-blocks of query heads
    constexpr int kMB = kD / 16;      // m-blocks of the head dimension (PV)
    constexpr int kKS = kD / 16;      // k-steps of the QK contraction

    // Fixed shared-memory offsets of this thread's K and V reads.
    uint32_t k_off[2][kD / 64];       // FP8: rows tau(g), 8+tau(g); chunks c, 4+c
    uint32_t v_off[4];                // FP8: rows tau(2c), tau(2c+1), 8+.., 8+..; chunk g
    if constexpr (kFp8) {
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
            for (int part = 0; part < kD / 64; ++part)
                k_off[half][part] = swz<C::kRowBytes, C::kSwizzle>(row0 + 8 * half + tau(g),
                                                                   16 * (4 * part + c));
        const int vr[4] = {row0 + tau(2 * c), row0 + tau(2 * c + 1), row0 + 8 + tau(2 * c),
                           row0 + 8 + tau(2 * c + 1)};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            v_off[i] = swz<C::kRowBytes, C::kSwizzle>(vr[i], (kD == 128 ? 16 : 8) * g);
    }

    // This warp's query rows of a segment as raw words: FP8, per n-block and
    // 64-dim part the 16 bf16 dims [16c, 16c+16) (8 words); BF16, the two
    // B-operand words of each k-step.  Heads past the group read as zero.
    constexpr int kQWords = C::kQWords;
    auto load_q = [&](const Segment& sg, uint32_t (&w)[kQWords]) {
        const int64_t hw0 = static_cast<int64_t>(sg.b) * a.num_q_heads + sg.h * IQ + kvh_w * G;
#pragma unroll
        for (int nb = 0; nb < kNB; ++nb) {
            const int hh = g + 8 * nb;
            const bool valid = hh < G;
            const uint16_t* qrow = a.q + (hw0 + (valid ? hh : 0)) * kD;
            if constexpr (kFp8) {
#pragma unroll
                for (int part = 0; part < kD / 64; ++part) {
                    const uint4* src = reinterpret_cast<const uint4*>(qrow + part * 64 + 16 * c);
                    const uint4 w0 = src[0], w1 = src[1];
                    uint32_t* d = &w[(nb * (kD / 64) + part) * 8];
                    d[0] = valid ? w0.x : 0u; d[1] = valid ? w0.y : 0u;
                    d[2] = valid ? w0.z : 0u; d[3] = valid ? w0.w : 0u;
                    d[4] = valid ? w1.x : 0u; d[5] = valid ? w1.y : 0u;
                    d[6] = valid ? w1.z : 0u; d[7] = valid ? w1.w : 0u;
                }
            } else {
#pragma unroll
                for (int j = 0; j < kKS; ++j) {
                    const uint32_t* src = reinterpret_cast<const uint32_t*>(qrow + 16 * j + 2 * c);
                    w[(nb * kKS + j) * 2 + 0] = valid ? src[0] : 0u;
                    w[(nb * kKS + j) * 2 + 1] = valid ? src[4] : 0u;
                }
            }
        }
        return (a.abort != nullptr) ? static_cast<int>(a.abort[sg.b]) : 0;
    };

    // A segment's query words and abort flag are loaded before the previous
    // segment's epilogue (C::kEarlyQ), which hides their latency behind it.
    uint32_t it = 0;
    uint32_t qw[kQWords];
    Segment s;
    bool have = walk.next(s);
    int aborted = 0;
    if constexpr (C::kEarlyQ) aborted = have ? load_q(s, qw) : 0;
    while (have) {
        Segment sn;
        const bool have_next = walk.next(sn);
        if constexpr (!C::kEarlyQ) aborted = load_q(s, qw);
        // (the item's indices are recomputed where they are used, after the
        // chunk loop, rather than held in registers through it)
        auto item_of = [&]() { return s.b * IPR + s.h; };
        auto whole_of = [&]() { return s.c0 == 0 && s.c1 == s.n; };
        auto slot_of = [&]() { return static_cast<int64_t>(blockIdx.x) + item_of(); };
        auto head0_of = [&]() {   // the item's first query-head row
            return static_cast<int64_t>(s.b) * a.num_q_heads + s.h * IQ;
        };
        // Cluster mode: a partial segment goes to a shared-memory record.  Of
        // a contiguous range only the first segment can start inside its item
        // (c0 > 0), and a partial segment that starts at its item's beginning
        // ends inside it and is the range's last: the former uses the
        // dedicated buffer (record 0), the latter the stage after its last
        // chunk (record 1; no stage is in use any more).  `it` must be the
        // chunk count after the segment.
        auto record = [&]() -> float* {
            const bool first = s.c0 > 0;
            float* r = first ? rec0 : reinterpret_cast<float*>(smem + (it % S) * C::kStageBytes);
            if (tid == 0) {
                scratch[first ? 5 : 6] = item_of();
                if (!first) scratch[7] = static_cast<int>(smem_addr(r));
            }
            return r;
        };

        if (aborted) {
            const bool whole = whole_of();
            const int64_t head0 = head0_of();
            // partial O and (m, l, lr) of the item: workspace slot or record
            float* o_dst = nullptr;
            float* ml_dst = nullptr;
            if (!whole) {
                if (a.cluster_size > 0) {
                    o_dst = record();
                    ml_dst = o_dst + C::kRecHeads * kD;
                } else {
                    o_dst = a.ws_o + slot_of() * IQ * kD;
                    ml_dst = a.ws_ml + slot_of() * IQ * 4;
                }
            }
            for (int e = tid; e < IQ * kD; e += kConsumerThreads) {
                const int hq = e / kD, d = e % kD;
                if (whole) {
                    a.out[(head0 + hq) * kD + d] = 0;
                    if (d == 0) a.lse[head0 + hq] = kNegInf;
                } else {
                    o_dst[hq * kD + d] = 0.f;
                    if (d == 0)
                        *reinterpret_cast<float4*>(ml_dst + 4 * hq) = make_float4(kNegInf, -1.f, -1.f, 0.f);
                }
            }
            if constexpr (C::kEarlyQ) aborted = have_next ? load_q(sn, qw) : 0;
            s = sn;
            have = have_next;
            continue;
        }

        // ---- Q^T as the B operand: column n = head g (+8 per n-block) -----
        uint32_t qb[kNB][kKS][2];
        float qs[kNB][2];   // score scale of S columns 2c and 2c+1
#pragma unroll
        for (int nb = 0; nb < kNB; ++nb) {
            float my_scale;
            if constexpr (kFp8) {
                // word j of the B operand holds dims D_c[4j..4j+3] of the
                // permuted contraction: this thread's dims in order
                float v[kD / 4];
#pragma unroll
                for (int k = 0; k < kD / 8; ++k) {
                    const uint32_t w = qw[nb * (kD / 8) + k];
                    v[2 * k] = bf16_bits_to_f32(w & 0xFFFFu);
                    v[2 * k + 1] = bf16_bits_to_f32(w >> 16);
                }
                float amax = 0.f;
#pragma unroll
                for (int k = 0; k < kD / 4; ++k) amax = fmaxf(amax, fabsf(v[k]));
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
                // 2^shift brings amax into [128, 256): with amax = f 2^e,
                // f in [0.5, 1), shift = 8 - e, where e comes from the
                // exponent field (a subnormal amax reads as e = -126, which
                // the clamp maps to the same shift as its true exponent)
                int shift = 0;
                if (amax > 0.f && isfinite(amax)) {
                    const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 126;
                    shift = min(60, max(-126, 8 - e));
                }
                // scaling by an exact power of two rounds like ldexp
                const float up = __uint_as_float(static_cast<uint32_t>(shift + 127) << 23);
#pragma unroll
                for (int j = 0; j < kKS; ++j) {
                    qb[nb][j][0] = pack_f16x2(v[4 * j] * up, v[4 * j + 1] * up);
                    qb[nb][j][1] = pack_f16x2(v[4 * j + 2] * up, v[4 * j + 3] * up);
                }
                my_scale = a.qk_scale * __uint_as_float(static_cast<uint32_t>(127 - shift) << 23);
            } else {
#pragma unroll
                for (int j = 0; j < kKS; ++j) {
                    qb[nb][j][0] = qw[(nb * kKS + j) * 2 + 0];
                    qb[nb][j][1] = qw[(nb * kKS + j) * 2 + 1];
                }
                my_scale = a.qk_scale;
            }
            // column 2c + col of this n-block is head 2c + col, owned by lanes 4(2c+col)+*
            qs[nb][0] = __shfl_sync(0xffffffffu, my_scale, 4 * (2 * c));
            qs[nb][1] = __shfl_sync(0xffffffffu, my_scale, 4 * (2 * c + 1));
        }

        float o[kNB][kMB][4];
#pragma unroll
        for (int nb = 0; nb < kNB; ++nb)
#pragma unroll
            for (int mb = 0; mb < kMB; ++mb) o[nb][mb][0] = o[nb][mb][1] = o[nb][mb][2] = o[nb][mb][3] = 0.f;
        // l: sum of the fp32 weights (for the LSE); lr: sum of the weights as
        // rounded for the PV product (the output's normaliser, so that the
        // output is a weighted mean with exactly the weights the MMA used)
        float m[kNB][2], l[kNB][2], lr[kNB][2];
#pragma unroll
        for (int nb = 0; nb < kNB; ++nb) {
            m[nb][0] = m[nb][1] = kNegInf;
            l[nb][0] = l[nb][1] = 0.f;
            lr[nb][0] = lr[nb][1] = 0.f;
        }
        int poisoned = 0;

        for (int ch = s.c0; ch < s.c1; ++ch, ++it) {
            const int stage = it % S;
            wait_or_give_up(&full_bar[stage], (it / S) & 1, cta_failed, a.ws_status);
            poisoned |= stage_bad_rd[stage];
            const int n_valid = min(kChunkTokens, s.L - ch * kChunkTokens);
            const bool tail = n_valid < kChunkTokens;
            const uint32_t kb_head = smem_addr(smem + stage * C::kStageBytes) + kvh_w * C::kHeadTileBytes;
            const uint32_t vb_head = kb_head + C::kTileBytes;
#pragma unroll
            for (int t = 0; t < kH; ++t) {
            const int rb = row0 + 16 * t;
            // FP8 offsets are relative to the warp's first tile; 16 rows on, the
            // swizzle pattern repeats, so the next tile is a plain offset
            const uint32_t kb = kb_head + (kFp8 ? t * 16 * C::kRowBytes : 0);
            const uint32_t vb = vb_head + (kFp8 ? t * 16 * C::kRowBytes : 0);

            // ---- S[16 tokens][8 heads] = K Q^T, two accumulator chains ------
            float acc[kNB][2][4];
#pragma unroll
            for (int nb = 0; nb < kNB; ++nb)
#pragma unroll
                for (int q = 0; q < 2; ++q) acc[nb][q][0] = acc[nb][q][1] = acc[nb][q][2] = acc[nb][q][3] = 0.f;
            if constexpr (kFp8) {
                uint32_t wa[kKS], wb[kKS];
#pragma unroll
                for (int part = 0; part < kD / 64; ++part) {
                    const uint4 x = lds128(kb + k_off[0][part]);
                    const uint4 y = lds128(kb + k_off[1][part]);
                    wa[4 * part + 0] = x.x; wa[4 * part + 1] = x.y; wa[4 * part + 2] = x.z; wa[4 * part + 3] = x.w;
                    wb[4 * part + 0] = y.x; wb[4 * part + 1] = y.y; wb[4 * part + 2] = y.z; wb[4 * part + 3] = y.w;
                }
#pragma unroll
                for (int j = 0; j < kKS; ++j) {
                    uint32_t a0, a2, a1, a3;
                    e4m3x4_to_f16x2x2(wa[j], a0, a2);   // token row tau(g): k 2c.. / 2c+8..
                    e4m3x4_to_f16x2x2(wb[j], a1, a3);   // token row 8+tau(g)
#pragma unroll
                    for (int nb = 0; nb < kNB; ++nb)
                        mma_f16(acc[nb][j & 1], a0, a1, a2, a3, qb[nb][j][0], qb[nb][j][1]);
                }
            } else {
                const int q8 = lane >> 3;
                const int row = rb + 8 * (q8 & 1) + (lane & 7);
#pragma unroll
                for (int j = 0; j < kKS; ++j) {
                    const int chunk16 = 2 * j + (q8 >> 1);
                    const uint32_t addr = kb + (chunk16 >> 3) * C::kSubTileBytes +
                                          swz<128, 128>(row, (chunk16 & 7) * 16);
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4(addr, a0, a1, a2, a3);
#pragma unroll
                    for (int nb = 0; nb < kNB; ++nb)
                        mma_bf16(acc[nb][j & 1], a0, a1, a2, a3, qb[nb][j][0], qb[nb][j][1]);
                }
            }

            // ---- online softmax over the 16 tokens, per head (log2 units) ----
            // p[nb][0..1]: token row g, heads 2c, 2c+1; p[nb][2..3]: row g + 8
            float p[kNB][4];
#pragma unroll
            for (int nb = 0; nb < kNB; ++nb)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    p[nb][i] = (acc[nb][0][i] + acc[nb][1][i]) * qs[nb][i & 1];
            if (tail) {
                const int t_lo = kFp8 ? rb + tau(g) : rb + g;
                const int t_hi = t_lo + 8;
#pragma unroll
                for (int nb = 0; nb < kNB; ++nb) {
                    if (t_lo >= n_valid) p[nb][0] = p[nb][1] = kNegInf;
                    if (t_hi >= n_valid) p[nb][2] = p[nb][3] = kNegInf;
                }
            }
            // Lazy rescaling: the running max m (uniform over the warp, per head)
            // only moves when some score exceeds it by more than the threshold;
            // until then p = 2^(s - m) <= 2^8 and no cross-lane max is needed.
            bool need = false;
#pragma unroll
            for (int nb = 0; nb < kNB; ++nb)
#pragma unroll
                for (int col = 0; col < 2; ++col)
                    need |= fmaxf(p[nb][col], p[nb][col + 2]) > m[nb][col] + kRescaleThreshold;
            if (__any_sync(0xffffffffu, need)) {
#pragma unroll
                for (int nb = 0; nb < kNB; ++nb) {
                    float alpha[2];
#pragma unroll
                    for (int col = 0; col < 2; ++col) {
                        float v = fmaxf(p[nb][col], p[nb][col + 2]);
                        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                        const float nm = fmaxf(m[nb][col], v);
                        alpha[col] = (nm == kNegInf) ? 1.f : exp2f(m[nb][col] - nm);
                        m[nb][col] = nm;
                        l[nb][col] *= alpha[col];
                        lr[nb][col] *= alpha[col];
                    }
#pragma unroll
                    for (int mb = 0; mb < kMB; ++mb) {
                        o[nb][mb][0] *= alpha[0];
                        o[nb][mb][1] *= alpha[1];
                        o[nb][mb][2] *= alpha[0];
                        o[nb][mb][3] *= alpha[1];
                    }
                }
            }
            // P^T as the PV B operand: k = token row, n = head g
            uint32_t pb[kNB][2];
#pragma unroll
            for (int nb = 0; nb < kNB; ++nb) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float ref = (m[nb][i & 1] == kNegInf) ? 0.f : m[nb][i & 1];
                    p[nb][i] = ex2_approx(p[nb][i] - ref);
                }
                l[nb][0] += p[nb][0] + p[nb][2];
                l[nb][1] += p[nb][1] + p[nb][3];
                uint32_t h01, h23;
                float r0, r1, r2, r3;
                if constexpr (kFp8) {
                    h01 = pack_f16x2(p[nb][0], p[nb][1]);
                    h23 = pack_f16x2(p[nb][2], p[nb][3]);
                    f16x2_nonneg_scaled(h01, r0, r1);   // (x 2^-112)
                    f16x2_nonneg_scaled(h23, r2, r3);
                    lr[nb][0] = fmaf(r0 + r2, 0x1p112f, lr[nb][0]);
                    lr[nb][1] = fmaf(r1 + r3, 0x1p112f, lr[nb][1]);
                } else {
                    h01 = pack_bf16x2(p[nb][0], p[nb][1]);
                    h23 = pack_bf16x2(p[nb][2], p[nb][3]);
                    bf16x2_to_f32x2(h01, r0, r1);
                    bf16x2_to_f32x2(h23, r2, r3);
                    lr[nb][0] += r0 + r2;
                    lr[nb][1] += r1 + r3;
                }
                pb[nb][0] = movmatrix_trans(h01);
                pb[nb][1] = movmatrix_trans(h23);
            }

            // ---- O^T[16 dims][8 heads] += V^T P^T per m-block of dims --------
            if constexpr (kFp8) {
                constexpr int kW = kD / 32;   // 32-bit words per thread and row: 4 (D=128), 2 (D=64)
                uint32_t x[4][kW];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    if constexpr (kW == 4) {
                        const uint4 t = lds128(vb + v_off[r]);
                        x[r][0] = t.x; x[r][1] = t.y; x[r][2] = t.z; x[r][3] = t.w;
                    } else {
                        const uint2 t = lds64(vb + v_off[r]);
                        x[r][0] = t.x; x[r][1] = t.y;
                    }
                }
                if (tail) {
                    const int vr[4] = {rb + tau(2 * c), rb + tau(2 * c + 1), rb + 8 + tau(2 * c),
                                       rb + 8 + tau(2 * c + 1)};
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        if (vr[r] >= n_valid)
#pragma unroll
                            for (int q = 0; q < kW; ++q) x[r][q] = 0u;
                }
#pragma unroll
                for (int q = 0; q < kW; ++q) {
                    // word q holds dims 4q..4q+3 of this thread's block: m-blocks 2q, 2q+1
                    uint32_t a0, a1, a2, a3;
                    e4m3x4_to_f16x2x2(prmt(x[0][q], x[1][q], 0x5140u), a0, a1);
                    e4m3x4_to_f16x2x2(prmt(x[2][q], x[3][q], 0x5140u), a2, a3);
#pragma unroll
                    for (int nb = 0; nb < kNB; ++nb)
                        mma_f16(o[nb][2 * q], a0, a1, a2, a3, pb[nb][0], pb[nb][1]);
                    e4m3x4_to_f16x2x2(prmt(x[0][q], x[1][q], 0x7362u), a0, a1);
                    e4m3x4_to_f16x2x2(prmt(x[2][q], x[3][q], 0x7362u), a2, a3);
#pragma unroll
                    for (int nb = 0; nb < kNB; ++nb)
                        mma_f16(o[nb][2 * q + 1], a0, a1, a2, a3, pb[nb][0], pb[nb][1]);
                }
            } else {
                const int q8 = lane >> 3;
                const int row = rb + 8 * (q8 >> 1) + (lane & 7);
                const int t0 = rb + 2 * c;    // tokens of a0/a1: t0, t0+1; of a2/a3: t0+8, t0+9
                uint32_t keep01 = 0xFFFFFFFFu, keep23 = 0xFFFFFFFFu;
                if (tail) {
                    keep01 = (t0 < n_valid ? 0x0000FFFFu : 0u) | (t0 + 1 < n_valid ? 0xFFFF0000u : 0u);
                    keep23 = (t0 + 8 < n_valid ? 0x0000FFFFu : 0u) | (t0 + 9 < n_valid ? 0xFFFF0000u : 0u);
                }
#pragma unroll
                for (int mb = 0; mb < kMB; ++mb) {
                    const int chunk16 = 2 * mb + (q8 & 1);
                    const uint32_t addr = vb + (chunk16 >> 3) * C::kSubTileBytes +
                                          swz<128, 128>(row, (chunk16 & 7) * 16);
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_trans(addr, a0, a1, a2, a3);
                    if (tail) {
                        a0 &= keep01; a1 &= keep01; a2 &= keep23; a3 &= keep23;
                    }
#pragma unroll
                    for (int nb = 0; nb < kNB; ++nb)
                        mma_bf16(o[nb][mb], a0, a1, a2, a3, pb[nb][0], pb[nb][1]);
                }
            }
            }   // tiles
            __syncwarp();
            if (lane == 0 && !(C::kRedInStage && ch + 1 == s.c1)) mbar_arrive(&empty_bar[stage]);
        }
        // the next segment's query words and abort flag, consumed after the
        // epilogue
        int next_aborted = 0;
        if constexpr (C::kEarlyQ) next_aborted = have_next ? load_q(sn, qw) : 0;
        const bool whole = whole_of();
        const int64_t head0 = head0_of();

        const int last_stage = (it + S - 1) % S;   // stage of the segment's last chunk
        float* red_o = C::kRedInStage ? reinterpret_cast<float*>(smem + last_stage * C::kStageBytes)
                                      : red_o_own;
        if constexpr (C::kRedInStage) {
            // every warp has finished reading the last chunk before O overwrites it
            named_barrier_sync(1, kConsumerThreads);
        }

        // ---- epilogue: combine the warps of each KV head, then write ------
#pragma unroll
        for (int nb = 0; nb < kNB; ++nb)
#pragma unroll
            for (int col = 0; col < 2; ++col) {
                float v = l[nb][col], vr = lr[nb][col];
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                vr += __shfl_xor_sync(0xffffffffu, vr, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                vr += __shfl_xor_sync(0xffffffffu, vr, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 16);
                vr += __shfl_xor_sync(0xffffffffu, vr, 16);
                l[nb][col] = v;
                lr[nb][col] = vr;
            }
        if (g == 0) {
#pragma unroll
            for (int nb = 0; nb < kNB; ++nb)
#pragma unroll
                for (int col = 0; col < 2; ++col) {
                    red_m[warp * kGP + 8 * nb + 2 * c + col] = m[nb][col];
                    red_l[warp * kGP + 8 * nb + 2 * c + col] = l[nb][col];
                    red_lr[warp * kGP + 8 * nb + 2 * c + col] = lr[nb][col];
                }
        }
        // O into red_o[warp][head][kD] (fp32); the 16-byte units of a row are
        // XOR-swizzled by red_swizzle of the row's head pair, which makes
        // these writes and the row-contiguous reads below conflict-free.
        {
            const uint32_t sw = red_swizzle<kFp8, kD>(c);
#pragma unroll
            for (int nb = 0; nb < kNB; ++nb)
#pragma unroll
                for (int col = 0; col < 2; ++col) {
                    float* row = red_o + (warp * kGP + 8 * nb + 2 * c + col) * kD;
                    if constexpr (kFp8) {
                        // dims [kD/8 g, kD/8 (g+1)): m-block mb holds dims
                        // 2mb (accumulator col) and 2mb + 1 (col + 2)
#pragma unroll
                        for (int k = 0; k < kD / 32; ++k) {
                            const uint32_t u = (kD / 32) * g + k;
                            *reinterpret_cast<float4*>(row + 4 * (u ^ sw)) =
                                make_float4(o[nb][2 * k][col], o[nb][2 * k][col + 2],
                                            o[nb][2 * k + 1][col], o[nb][2 * k + 1][col + 2]);
                        }
                    } else {
                        // m-block mb holds dims 16mb + g (col) and 16mb + g + 8 (col + 2)
#pragma unroll
                        for (int mb = 0; mb < kMB; ++mb) {
                            const uint32_t d_lo = 16 * mb + g, d_hi = d_lo + 8;
                            row[4 * ((d_lo >> 2) ^ sw) + (d_lo & 3)] = o[nb][mb][col];
                            row[4 * ((d_hi >> 2) ^ sw) + (d_hi & 3)] = o[nb][mb][col + 2];
                        }
                    }
                }
        }
        named_barrier_sync(1, kConsumerThreads);
        // Thread -> (head, 16-byte unit of dims): per pass the consumer
        // threads cover kConsumerThreads / (kD/4) heads.
        {
            float* o_dst = nullptr;    // partial O and (m, l, lr): workspace slot or record
            float* ml_dst = nullptr;
            if (!whole) {
                if (a.cluster_size > 0) {
                    o_dst = record();
                    ml_dst = o_dst + C::kRecHeads * kD;
                } else {
                    o_dst = a.ws_o + slot_of() * IQ * kD;
                    ml_dst = a.ws_ml + slot_of() * IQ * 4;
                }
            }
            constexpr int kUnits = kD / 4;
            constexpr int kHeadsPerPass = kConsumerThreads / kUnits;
            const int u = tid % kUnits;
            for (int hq = tid / kUnits; hq < IQ; hq += kHeadsPerPass) {
                const int kvh = hq / G;
                const int hl = hq - kvh * G;                 // head within its KV head's group
                const int r0 = kvh * kWarpsPerHead * kGP + hl;   // its row in the first warp
                const uint32_t su = u ^ red_swizzle<kFp8, kD>((hl & 7) >> 1);
                float M = kNegInf;
#pragma unroll
                for (int w = 0; w < kWarpsPerHead; ++w) M = fmaxf(M, red_m[r0 + w * kGP]);
                float Lsum = 0.f, Lr = 0.f;
                float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int w = 0; w < kWarpsPerHead; ++w) {
                    const float mw = red_m[r0 + w * kGP];
                    const float wt = (mw == kNegInf) ? 0.f : exp2f(mw - M);
                    Lsum += wt * red_l[r0 + w * kGP];
                    Lr += wt * red_lr[r0 + w * kGP];
                    const float4 x = *reinterpret_cast<const float4*>(red_o + (r0 + w * kGP) * kD + 4 * su);
                    O.x += wt * x.x;
                    O.y += wt * x.y;
                    O.z += wt * x.z;
                    O.w += wt * x.w;
                }
                const int64_t hrow = head0 + hq;
                if (whole) {
                    uint32_t* dst = reinterpret_cast<uint32_t*>(a.out + hrow * kD + 4 * u);
                    if (poisoned) {
                        dst[0] = 0u;
                        dst[1] = 0u;
                        if (u == 0) a.lse[hrow] = kNegInf;
                    } else {
                        const float k = a.v_scale / Lr;
                        dst[0] = pack_bf16x2(O.x * k, O.y * k);
                        dst[1] = pack_bf16x2(O.z * k, O.w * k);
                        if (u == 0) a.lse[hrow] = (M + log2f(Lsum)) * kLn2;
                    }
                } else {
                    const float4 val = poisoned ? make_float4(0.f, 0.f, 0.f, 0.f)
                                                : make_float4(O.x * a.v_scale, O.y * a.v_scale,
                                                              O.z * a.v_scale, O.w * a.v_scale);
                    *reinterpret_cast<float4*>(o_dst + hq * kD + 4 * u) = val;
                    if (u == 0)
                        *reinterpret_cast<float4*>(ml_dst + 4 * hq) =
                            poisoned ? make_float4(kNegInf, -1.f, -1.f, 0.f)
                                     : make_float4(M, Lsum, Lr, 0.f);
                }
            }
        }
        // the stage is about to be refilled by TMA (async proxy) after our
        // generic-proxy writes to it: order them first
        if constexpr (C::kRedInStage) fence_proxy_async_smem();
        named_barrier_sync(1, kConsumerThreads);
        if (C::kRedInStage && lane == 0) mbar_arrive(&empty_bar[last_stage]);
        if constexpr (C::kEarlyQ) aborted = next_aborted;
        s = sn;
        have = have_next;
    }
    if (a.cluster_size > 0) attn_cluster_reduce<kFp8, kD, kGP, kH>(a, smem);
}

// ---------------------------------------------------------------------------
// merge: per (request, KV head) item, one CTA for all of its query heads
// (kHPC = 16) or, when the items are split over many CTAs, one CTA per group
// of 4 query heads (kHPC = 4: each thread then owns a single output and has
// every segment's value in flight at once).  For each query head h of the
// item: M = max_s m_s, L = sum_s l_s 2^(m_s - M), Lr = sum_s lr_s 2^(m_s - M),
// out = sum_s O_s 2^(m_s - M) / Lr and lse = M + log2 L (natural units) over the
// item's segments s (one per CTA that worked on it); lr is the sum of the
// weights as rounded for the PV product, l of the fp32 weights.  Segment
// weights are computed once into shared memory (in tiles of kMergeTile
// segments, merged online), then every thread sums its (head, dim) outputs
// with independent loads.
// ---------------------------------------------------------------------------
constexpr int kMergeThreads = 512;
constexpr int kMergeTile = 128;
constexpr int kMergeFastSegs = 8;   // items split over at most this many CTAs: one round trip

__device__ __forceinline__ int64_t cta_of_unit(int64_t u, int64_t U, int N) {
    // largest c with floor(c * U / N) <= u
    return ((u + 1) * N + U - 1) / U - 1;
}

template <int kD, int kHPC>
__global__ void __launch_bounds__(kMergeThreads)
attn_merge_kernel(const AttnArgs a) {
    __shared__ float s_w[kMergeTile][kHPC];   // m_s, then weight 2^(m_s - M), of segment s, head h
    __shared__ float s_l[kMergeTile][kHPC];   // l_s (fp32 weights)
    __shared__ float s_lr[kMergeTile][kHPC];  // lr_s (weights as rounded for the PV product)
    __shared__ float s_m[kHPC], s_sum[kHPC], s_sumr[kHPC], s_scale[kHPC];
    __shared__ int s_dead;
    __shared__ int s_red[2][kMergeThreads / 32], s_nb, s_nc;
    launch_dependents();
    const int tid = threadIdx.x;
    constexpr int kGroups = 16 / kHPC;       // CTAs per item
    const int IPR = a.items_per_req;
    const int item = blockIdx.x / kGroups;
    const int b = item / IPR, h = item % IPR;
    const int G = a.group * a.kv_per_item;   // query heads of one item (at most 16)
    const int hq0 = (blockIdx.x % kGroups) * kHPC;   // this CTA's first head of the item
    if (hq0 >= G) return;
    const int NH = min(kHPC, G - hq0);       // this CTA's heads
    const int64_t head0 = static_cast<int64_t>(b) * a.num_q_heads + h * G + hq0;
    // Shared-prefix mode: the chunk begins come from the plan kernels, which
    // precede the partial kernel.
    if (a.chunk_begin != nullptr) grid_dependency_wait();
    // Unit counts (chunks from the request's first) of the requests before b,
    // of b and of the batch, from the lengths (an input no kernel writes),
    // before the grid-dependency wait: this overlaps the partial kernel's tail.
    {
        const int64_t max_tokens = static_cast<int64_t>(a.max_pages) * a.page_size;
        int pre_part = 0, tot_part = 0;
        for (int bb = tid; bb < a.batch; bb += kMergeThreads) {
            const int32_t len = a.seq_lens[bb];
            int nb = (len >= 1 && static_cast<int64_t>(len) <= max_tokens)
                         ? (len + kChunkTokens - 1) / kChunkTokens
                         : 0;
            const int nc = nb;
            if (nb > 0 && a.chunk_begin != nullptr) nb -= a.chunk_begin[bb];
            if (bb == b) s_nc = nc;
            tot_part += nb;
            if (bb < b) pre_part += nb;
            if (bb == b) s_nb = nb;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            pre_part += __shfl_xor_sync(0xffffffffu, pre_part, off);
            tot_part += __shfl_xor_sync(0xffffffffu, tot_part, off);
        }
        if ((tid & 31) == 0) {
            s_red[0][tid >> 5] = pre_part;
            s_red[1][tid >> 5] = tot_part;
        }
        __syncthreads();
    }
    int32_t pre = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kMergeThreads / 32; ++w) {
        pre += s_red[0][w];
        tot += s_red[1][w];
    }
    const int32_t n = s_nb;
    grid_dependency_wait();
    if (n == 0 && s_nc > 0) return;   // finished by the shared-prefix pass
    if (n == 0) {
        for (int e = tid; e < NH * kD; e += kMergeThreads) {
            const int hq = e / kD, d = e % kD;
            a.out[(head0 + hq) * kD + d] = 0;
            if (d == 0) a.lse[head0 + hq] = kNegInf;
        }
        return;
    }
    const int64_t U = static_cast<int64_t>(IPR) * tot;
    const int NE = static_cast<int>(U < a.num_ctas ? U : a.num_ctas);   // as in the partial kernel
    const int64_t u0 = static_cast<int64_t>(IPR) * pre + static_cast<int64_t>(h) * n;
    const int64_t c0 = cta_of_unit(u0, U, NE);
    const int64_t c1 = cta_of_unit(u0 + n - 1, U, NE);
    // the shared-prefix pass's record of this item, if it has one: one more
    // segment, after the CTAs' ones
    const int pfx = (a.chunk_begin != nullptr && a.chunk_begin[b] > 0) ? 1 : 0;
    if (c0 == c1 && pfx == 0) return;   // finished by the partial kernel
    const int nseg = static_cast<int>(c1 - c0 + 1);
    const int ntot = nseg + pfx;
    const int64_t stride = static_cast<int64_t>(G) * kD;
    if (ntot <= kMergeFastSegs) {
        // Few segments: thread -> (head, 4 dims); every segment's (m, l, lr)
        // and output quad are requested at once (one round trip).
        constexpr int kQuads = kD / 4;
        const int hq = tid / kQuads, q = tid - hq * kQuads;
        if (hq >= NH) return;
        float4 ml[kMergeFastSegs], x[kMergeFastSegs];
#pragma unroll
        for (int k = 0; k < kMergeFastSegs; ++k) {
            if (k < ntot) {
                const int64_t slot = c0 + k + item;
                const float* mp = k < nseg ? a.ws_ml + (slot * G + hq0 + hq) * 4
                                           : a.pfx_ml + (static_cast<int64_t>(item) * G + hq0 + hq) * 4;
                const float* op = (k < nseg ? a.ws_o + slot * stride : a.pfx_o + item * stride) +
                                  static_cast<int64_t>(hq0 + hq) * kD + 4 * q;
                ml[k] = *reinterpret_cast<const float4*>(mp);
                x[k] = *reinterpret_cast<const float4*>(op);
            }
        }
        float M = kNegInf;
        int dead = 0;
#pragma unroll
        for (int k = 0; k < kMergeFastSegs; ++k) {
            if (k < ntot) {
                M = fmaxf(M, ml[k].x);
                dead |= ml[k].y < 0.f;
            }
        }
        float Lsum = 0.f, Lr = 0.f;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < kMergeFastSegs; ++k) {
            if (k < ntot) {
                const float wt = (ml[k].x == kNegInf) ? 0.f : exp2f(ml[k].x - M);
                Lsum += wt * ml[k].y;
                Lr += wt * ml[k].z;
                O.x += wt * x[k].x;
                O.y += wt * x[k].y;
                O.z += wt * x[k].z;
                O.w += wt * x[k].w;
            }
        }
        uint32_t* dst = reinterpret_cast<uint32_t*>(a.out + (head0 + hq) * kD + 4 * q);
        if (dead) {
            dst[0] = 0u;
            dst[1] = 0u;
        } else {
            dst[0] = pack_bf16x2(O.x / Lr, O.y / Lr);
            dst[1] = pack_bf16x2(O.z / Lr, O.w / Lr);
        }
        if (q == 0) a.lse[head0 + hq] = dead ? kNegInf : (M + log2f(Lsum)) * kLn2;
        return;
    }
    if (tid < kHPC) {
        s_m[tid] = kNegInf;
        s_sum[tid] = 0.f;
        s_sumr[tid] = 0.f;
    }
    if (tid == 0) s_dead = 0;
    constexpr int kPer = (kHPC * kD + kMergeThreads - 1) / kMergeThreads;
    float acc[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) acc[k] = 0.f;

    // tiles of the CTAs' segments, then (shared-prefix mode) a tile of the
    // prefix record alone
    for (int t0 = 0; t0 < ntot;) {
        const bool ptile = t0 >= nseg;
        const int tn = ptile ? 1 : min(kMergeTile, nseg - t0);
        // (1) the tile's (m, l, lr) of this CTA's heads into shared memory:
        // one round trip
        for (int e = tid; e < tn * NH; e += kMergeThreads) {
            const int sg = e / NH, hq = e % NH;
            const int64_t slot = c0 + t0 + sg + item;
            const float* mp = ptile ? a.pfx_ml + (static_cast<int64_t>(item) * G + hq0 + hq) * 4
                                    : a.ws_ml + (slot * G + hq0 + hq) * 4;
            const float4 ml = *reinterpret_cast<const float4*>(mp);
            s_w[sg][hq] = ml.x;
            s_l[sg][hq] = ml.y;
            s_lr[sg][hq] = ml.z;
        }
        __syncthreads();
        // (2) per head, in shared memory: new running max, weights, sum
        for (int hq = tid >> 5; hq < NH; hq += kMergeThreads / 32) {
            float mx = kNegInf;
            int dead = 0;
            for (int sg = (tid & 31); sg < tn; sg += 32) {
                mx = fmaxf(mx, s_w[sg][hq]);
                dead |= s_l[sg][hq] < 0.f;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                dead |= __shfl_xor_sync(0xffffffffu, dead, off);
            }
            const float m_old = s_m[hq];
            const float m_new = fmaxf(m_old, mx);
            float lsum = 0.f, lrsum = 0.f;
            for (int sg = (tid & 31); sg < tn; sg += 32) {
                const float ms = s_w[sg][hq];
                const float wt = (ms == kNegInf) ? 0.f : exp2f(ms - m_new);
                s_w[sg][hq] = wt;
                lsum += wt * s_l[sg][hq];
                lrsum += wt * s_lr[sg][hq];
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
                lrsum += __shfl_xor_sync(0xffffffffu, lrsum, off);
            }
            if ((tid & 31) == 0) {
                const float r = (m_old == kNegInf) ? 0.f : exp2f(m_old - m_new);
                if (dead) s_dead = 1;
                s_scale[hq] = r;
                s_sum[hq] = s_sum[hq] * r + lsum;
                s_sumr[hq] = s_sumr[hq] * r + lrsum;
                s_m[hq] = m_new;
            }
        }
        __syncthreads();
        // (3) outputs: segment-major, kPer x kUnroll independent loads in flight
        const float* base = (ptile ? a.pfx_o + item * stride : a.ws_o + (c0 + t0 + item) * stride) +
                            static_cast<int64_t>(hq0) * kD;
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int e = tid + k * kMergeThreads;
            if (e < NH * kD) acc[k] *= s_scale[e / kD];
        }
        if constexpr (kPer == 1) {
            const int e = tid;
            if (e < NH * kD) {
                const int hq = e / kD;
#pragma unroll 16
                for (int sg = 0; sg < tn; ++sg) acc[0] += s_w[sg][hq] * base[sg * stride + e];
            }
        } else {
#pragma unroll 8
            for (int sg = 0; sg < tn; ++sg) {
#pragma unroll
                for (int k = 0; k < kPer; ++k) {
                    const int e = tid + k * kMergeThreads;
                    if (e < NH * kD) acc[k] += s_w[sg][e / kD] * base[sg * stride + e];
                }
            }
        }
        __syncthreads();
        t0 += tn;
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int e = tid + k * kMergeThreads;
        if (e >= NH * kD) break;
        const int hq = e / kD, d = e % kD;
        if (s_dead) {
            a.out[(head0 + hq) * kD + d] = 0;
            if (d == 0) a.lse[head0 + hq] = kNegInf;
        } else {
            a.out[(head0 + hq) * kD + d] = f32_to_bf16_bits(acc[k] / s_sumr[hq]);
            if (d == 0) a.lse[head0 + hq] = (s_m[hq] + log2f(s_sum[hq])) * kLn2;
        }
    }
}

// ---------------------------------------------------------------------------
// host-side dispatch
// ---------------------------------------------------------------------------
template <bool kFp8, int kD, int kGP, int kH>
static cudaError_t launch_variant(int grid, cudaStream_t stream, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const AttnArgs& args) {
    using C = AttnCfg<kFp8, kD, kGP, kH>;
    PdlLaunch l(dim3(grid), dim3(kAttnThreads), C::kSmemBytes, stream);
    if (args.cluster_size > 0) l.set_cluster(args.cluster_size);
    return cudaLaunchKernelEx(&l.cfg, attn_partial_kernel<kFp8, kD, kGP, kH>, tk, tv, args);
}

template <bool kFp8, int kD, int kGP, int kH>
static cudaError_t max_clusters_variant(int cluster_size, int* clusters) {
    using C = AttnCfg<kFp8, kD, kGP, kH>;
    auto* fn = attn_partial_kernel<kFp8, kD, kGP, kH>;
    cudaError_t e = cudaSuccess;
    if (cluster_size > 8) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cluster_size);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(cluster_size));
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaOccupancyMaxActiveClusters(clusters, fn, &cfg);
}

// (fp8, head_dim, group pad, KV heads per item)
#define PKV_FOR_EACH_VARIANT(X)                                                    \
    X(true, 64, 8, 1) X(true, 64, 16, 1) X(true, 128, 8, 1) X(true, 128, 16, 1)    \
    X(false, 64, 8, 1) X(false, 64, 16, 1) X(false, 128, 8, 1) X(false, 128, 16, 1) \
    X(true, 64, 8, 2) X(true, 128, 8, 2)

#define PKV_MATCH(F, D, GP, H) \
    (fp8 == F && head_dim == D && group_pad == GP && kv_per_item == H)

size_t attn_partial_smem_bytes(bool fp8, int head_dim, int group_pad, int kv_per_item) {
#define X(F, D, GP, H) \
    if (PKV_MATCH(F, D, GP, H)) return AttnCfg<F, D, GP, H>::kSmemBytes;
    PKV_FOR_EACH_VARIANT(X)
#undef X
    return 0;
}

cudaError_t attn_set_smem_attr(bool fp8, int head_dim, int group_pad, int kv_per_item) {
#define X(F, D, GP, H)                                                              \
    if (PKV_MATCH(F, D, GP, H))                                                      \
        return cudaFuncSetAttribute(attn_partial_kernel<F, D, GP, H>,                \
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,     \
                                    AttnCfg<F, D, GP, H>::kSmemBytes);
    PKV_FOR_EACH_VARIANT(X)
#undef X
    return cudaErrorInvalidValue;
}

cudaError_t attn_occupancy(bool fp8, int head_dim, int group_pad, int kv_per_item,
                           int* blocks_per_sm) {
#define X(F, D, GP, H)                                                               \
    if (PKV_MATCH(F, D, GP, H))                                                       \
        return cudaOccupancyMaxActiveBlocksPerMultiprocessor(                         \
            blocks_per_sm, attn_partial_kernel<F, D, GP, H>, kAttnThreads,            \
            AttnCfg<F, D, GP, H>::kSmemBytes);
    PKV_FOR_EACH_VARIANT(X)
#undef X
    return cudaErrorInvalidValue;
}

cudaError_t attn_max_clusters(bool fp8, int head_dim, int group_pad, int kv_per_item,
                              int cluster_size, int* clusters) {
#define X(F, D, GP, H) \
    if (PKV_MATCH(F, D, GP, H)) return max_clusters_variant<F, D, GP, H>(cluster_size, clusters);
    PKV_FOR_EACH_VARIANT(X)
#undef X
    return cudaErrorInvalidValue;
}

cudaError_t launch_attn_partial(bool fp8, int head_dim, int group_pad, int kv_per_item, int grid,
                                cudaStream_t stream, const CUtensorMap& tmap_k,
                                const CUtensorMap& tmap_v, const AttnArgs& args) {
#define X(F, D, GP, H) \
    if (PKV_MATCH(F, D, GP, H)) return launch_variant<F, D, GP, H>(grid, stream, tmap_k, tmap_v, args);
    PKV_FOR_EACH_VARIANT(X)
#undef X
    return cudaErrorInvalidValue;
}

cudaError_t launch_attn_merge(int head_dim, cudaStream_t stream, const AttnArgs& args) {
    // Items split over 8 or more CTAs on average (small batches on a full
    // grid) are merged by one CTA per 4 query heads, the others by one CTA
    // per item.
    const int64_t items = static_cast<int64_t>(args.batch) * args.items_per_req;
    const bool wide = args.num_ctas >= 8 * items;
    PdlLaunch l(dim3(static_cast<unsigned>(items * (wide ? 4 : 1))), dim3(kMergeThreads), 0, stream);
    if (head_dim == 64)
        return wide ? cudaLaunchKernelEx(&l.cfg, attn_merge_kernel<64, 4>, args)
                    : cudaLaunchKernelEx(&l.cfg, attn_merge_kernel<64, 16>, args);
    return wide ? cudaLaunchKernelEx(&l.cfg, attn_merge_kernel<128, 4>, args)
                : cudaLaunchKernelEx(&l.cfg, attn_merge_kernel<128, 16>, args);
}

}  // namespace pkv
