// prefix.cu -- the shared-prefix pass of FP8 paged decode attention for
// sm_100a: requests whose leading pages are the same physical pages attend
// to those pages once, together.
//
// Source pages: "大模型推理优化：量化、压缩与安全验证", section "保护共享 KV
// cache" (hundreds of requests read the same physical KV pages; cache reuse
// is one of the mechanisms that depend on it); remio.ai commentary, section
// "为什么 Cloudflare 的小型缓存胜过单纯的速度" (prefix caching reuses the state
// of identical prompt beginnings).  The pages give no kernel for it; the
// split here is exact: attention over a request's chunks is the log-sum-exp
// combination of attention over any partition of them, so the chunks a group
// of requests shares are attended in one pass for all members and combined
// with each member's own chunks by the merge kernel.
//
//  * Plan (four small kernels).  A request joins its predecessor's group
//    when the two share at least kPfxMinChunks leading 64-token chunks that
//    lie entirely before both newest tokens (same page ids, valid ids).  A
//    group's reference row is its member with the most such chunks; every
//    member's shared chunks are counted against it.  Groups are cut into
//    tiles of at most 64 / G consecutive members; a tile covers two KV heads
//    (one work item of the split-K kernel) and the largest shared count of
//    its members, read from the reference row.  chunk_begin[b] tells the
//    split-K kernels where request b's own chunks start (0 for requests in
//    no tile).
//  * Tile = one tcgen05 tensor-core tile of 128 rows: row = (member, KV head
//    of the pair, query head of the group), so the 64 / G members' queries of
//    both KV heads share every K/V byte read.  Per 64-token chunk: warp 4
//    streams the raw FP8 K and V rows of both heads (TMA, 128-byte swizzle);
//    warps 0-3 (thread = row = tensor-memory lane) convert K to f16 token
//    rows (exact), thread 0 issues S = Q K^T (M = 128, N = 128 tokens of both
//    heads, K = 128 dims) into tensor memory; then the warps convert V to
//    f16 token rows (the MN-major operand of the product, so no transpose);
//    each thread then reads its row of S (its own head's 64
//    columns), updates its online softmax and writes P (f16, the other head's
//    columns zero: the product is block-diagonal) back into tensor memory
//    over S; thread 0 issues O += P V (A = P from tensor memory, K = 128
//    tokens, N = 128 dims).  Q is scaled per row by a power of two so that
//    its f16 copy is exact, as in the split-K kernel.
//  * Each member row ends with a partial record (m, l, lr, O) in the
//    split-K kernels' record format, one per (request, item), which the
//    merge kernel combines with the records of the member's own chunks.
#include <climits>

#include "device.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace pkv {

namespace {

constexpr float kPfxLog2RescaleThreshold = 8.0f;
constexpr float kPfxNegInf = -__builtin_huge_valf();
constexpr float kPfxLn2 = 0.6931471805599453f;
constexpr int kPfxD = 128;
// shared memory: Q tile, converted K or V tile (token rows of 64-dim blocks),
// raw FP8 K and V of one chunk of both heads, barriers
constexpr int kPfxAtom = kPfxRows * 128;                 // 128 rows x 128 bytes: 64 f16 columns
constexpr int kPfxQOff = 0;                               // 2 atoms (dims 0-63, 64-127)
constexpr int kPfxKVOff = kPfxQOff + 2 * kPfxAtom;        // 2 atoms (dims 0-63, 64-127)
constexpr int kPfxRawBytes = 2 * kChunkTokens * kPfxD;   // one FP8 operand of both heads: 16 KiB
constexpr int kPfxRawKOff = kPfxKVOff + 2 * kPfxAtom;
constexpr int kPfxRawVOff = kPfxRawKOff + kPfxRawBytes;
constexpr int kPfxBarOff = kPfxRawVOff + kPfxRawBytes;
constexpr int kPfxXOff = kPfxBarOff + 64;
// The CTA holds two independent halves (a CTA that allocates tensor memory
// gets an SM to itself), each with its own 8 row warps, TMA warp, shared
// memory region and 256 tensor-memory columns.
constexpr int kPfxHalfBytes = (kPfxXOff + 3 * kPfxRowThreads * 4 + 1023) / 1024 * 1024;
constexpr int kPfxSmemBytes = 2 * kPfxHalfBytes + 1024;   // + alignment slack
constexpr int kPfxRowWarps = kPfxRowThreads / 32;
constexpr int kPfxHalfWarps = kPfxRowWarps + 1;
constexpr uint32_t kPfxTmemCols = 512;   // per half: S / P 128 columns, then O 128
constexpr uint32_t kPfxOCol = 128;

}  // namespace

// ---------------------------------------------------------------------------
// plan
// ---------------------------------------------------------------------------
namespace {

// Chunks of request b that lie entirely before its newest token (-1 if its
// length is invalid).
__device__ __forceinline__ int full_chunks(const PrefixArgs& a, int b) {
    const int64_t max_tokens = static_cast<int64_t>(a.max_pages) * a.page_size;
    const int32_t len = a.seq_lens[b];
    return (len >= 1 && len <= max_tokens) ? (len - 1) / kChunkTokens : -1;
}

// Leading chunks (at most `limit`) whose page ids are equal and valid in the
// page-table rows of requests b0 and b1; one warp.
__device__ __forceinline__ int common_chunks(const PrefixArgs& a, int b0, int b1, int limit, int lane) {
    const int pages = static_cast<int>((static_cast<int64_t>(limit) * kChunkTokens + a.page_size - 1) / a.page_size);
    const int32_t* r0 = a.page_table + static_cast<int64_t>(b0) * a.max_pages;
    const int32_t* r1 = a.page_table + static_cast<int64_t>(b1) * a.max_pages;
    int same = pages;
    for (int j0 = 0; j0 < pages; j0 += 32) {
        const int j = j0 + lane;
        bool ok = true;
        if (j < pages) {
            const int32_t p1 = r1[j], p0 = r0[j];
            ok = p1 == p0 && p1 >= 0 && p1 < a.num_pages;
        }
        const uint32_t bad = __ballot_sync(0xffffffffu, !ok);
        if (bad) {
            same = j0 + __ffs(bad) - 1;
            break;
        }
    }
    return min(limit, static_cast<int>(static_cast<int64_t>(same) * a.page_size / kChunkTokens));
}

}  // namespace

// Step 1 (one warp per request): link[b] = leading chunks request b shares
// with request b - 1 (chunks before both newest tokens; equal, valid page
// ids).  b joins b - 1's group when link[b] >= min_chunks.
__global__ void __launch_bounds__(256) prefix_link_kernel(const PrefixArgs a) {
    launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x * 8 + warp;
    if (b >= a.batch) return;
    int shared = 0;
    if (b > 0) {
        const int f1 = full_chunks(a, b), f0 = full_chunks(a, b - 1);
        if (f1 >= 0 && f0 >= 0) shared = common_chunks(a, b - 1, b, min(f1, f0), lane);
    }
    // the workspace may still be read by the previous call's kernels until
    // the dependency wait; the page table and lengths above are inputs no
    // kernel writes
    grid_dependency_wait();
    if (lane == 0) a.link[b] = shared;
    // the call's status word starts at zero (later kernels of the call only
    // set bits in it)
    if (b == 0 && lane == 0) *a.status = 0u;
}

// Step 2 (one CTA): leader[b] = first request of b's group (a scan for the
// last group start at or before b), then ref[b] = the group's reference row:
// its member with the most full chunks, the first of them on a tie.
__global__ void __launch_bounds__(kPfxPlanThreads) prefix_group_kernel(const PrefixArgs a) {
    __shared__ int s_w[kPfxPlanThreads / 32], s_carry, s_next;
    launch_dependents();
    grid_dependency_wait();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int B = a.batch;
    if (tid == 0) s_carry = 0;
    for (int b = tid; b < B; b += kPfxPlanThreads) a.refkey[b] = 0ull;
    __syncthreads();
    for (int base = 0; base < B; base += kPfxPlanThreads) {
        const int b = base + tid;
        // inclusive max-scan of "b starts a group ? b : -1"
        int l = (b < B && (b == 0 || a.link[b] < a.min_chunks)) ? b : -1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int pl = __shfl_up_sync(0xffffffffu, l, off);
            if (lane >= off) l = max(l, pl);
        }
        if (lane == 31) s_w[warp] = l;
        __syncthreads();
        if (warp == 0) {
            int w = s_w[lane];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int pw = __shfl_up_sync(0xffffffffu, w, off);
                if (lane >= off) w = max(w, pw);
            }
            int x = __shfl_up_sync(0xffffffffu, w, 1);
            if (lane == 0) x = -1;
            s_w[lane] = max(x, s_carry);
            if (lane == 31) s_next = max(w, s_carry);
        }
        __syncthreads();
        l = max(l, s_w[warp]);
        if (b < B) {
            a.leader[b] = l;
            const int f = full_chunks(a, b);
            // larger full-chunk count first, then the smaller index
            const unsigned long long key = (static_cast<unsigned long long>(f < 0 ? 0 : f + 1) << 32) |
                                           static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(b));
            atomicMax(&a.refkey[l], key);
        }
        __syncthreads();
        if (tid == 0) s_carry = s_next;
        __syncthreads();
    }
    for (int b = tid; b < B; b += kPfxPlanThreads)
        a.ref[b] = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(a.refkey[a.leader[b]] & 0xFFFFFFFFull));
}

// Step 3 (one warp per request): share[b] = leading chunks b shares with its
// group's reference row (0 for the reference itself and for requests alone).
__global__ void __launch_bounds__(256) prefix_share_kernel(const PrefixArgs a) {
    launch_dependents();
    grid_dependency_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x * 8 + warp;
    if (b >= a.batch) return;
    const int r = a.ref[b];
    int shared = 0;
    if (r != b) {
        const int f1 = full_chunks(a, b), f0 = full_chunks(a, r);
        if (f1 >= 0 && f0 >= 0) shared = common_chunks(a, r, b, min(f1, f0), lane);
    }
    if (lane == 0) a.share[b] = shared;
}

// Step 4 (one CTA): tiles.  Each run of members_per_tile consecutive members
// of a group (from its first request) is a tile if it has 2 members and one
// of them, not the reference, shares at least min_chunks chunks; the tile
// covers the largest share of those members, which the reference (if it is
// one of them) takes as its own.  chunk_begin[b] = b's chunks in a tile.
__global__ void __launch_bounds__(kPfxPlanThreads) prefix_tile_kernel(const PrefixArgs a) {
    __shared__ int s_count;
    launch_dependents();
    grid_dependency_wait();
    const int tid = threadIdx.x;
    const int B = a.batch, T = a.members_per_tile;
    if (tid == 0) s_count = 0;
    __syncthreads();
    for (int b = tid; b < B; b += kPfxPlanThreads) {
        const int lead = a.leader[b];
        if ((b - lead) % T != 0) continue;
        const int r = a.ref[b];
        int nm = 0, mx = 0;
        for (int k = 0; k < T && b + k < B; ++k) {
            if (a.leader[b + k] != lead) break;
            ++nm;
            if (b + k != r) mx = max(mx, a.share[b + k]);
        }
        const bool tile = nm >= 2 && mx >= a.min_chunks;
        if (tile) {
            const int t = atomicAdd(&s_count, 1);
            int32_t* d = a.tiles + 4 * t;
            d[0] = r;      // page-table row the tile reads
            d[1] = b;      // first member
            d[2] = nm;     // members
            d[3] = mx;     // chunks
        }
        for (int k = 0; k < nm; ++k) {
            const int m = b + k;
            const int ps = tile ? (m == r ? mx : a.share[m]) : 0;
            int cbeg = ps;
            if (tile) {
                // a member with few chunks after its shared ones is finished by
                // the tile itself
                const int n = full_chunks(a, m) + 1;
                if (n - ps <= a.tail_chunks) cbeg = n;
            }
            a.pshare[m] = ps;
            a.chunk_begin[m] = cbeg;
        }
    }
    __syncthreads();
    if (tid == 0) *a.num_tiles = s_count;
}

// ---------------------------------------------------------------------------
// the shared-prefix tile kernel
// ---------------------------------------------------------------------------
namespace {

// Byte offset of 16-byte chunk `j` (0-7) of row `r` in a 128-row atom with
// 128-byte rows and the 128-byte swizzle (the layout TMA writes and the
// tensor-core descriptors read).
__device__ __forceinline__ uint32_t atom_off(uint32_t r, uint32_t j) {
    return r * 128u + ((j ^ (r & 7u)) << 4);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// Boxes of chunk c that lie in the request's first `npages` pages (all of
// them except in the last chunk of a request with pages under 64 tokens).
__device__ __forceinline__ int chunk_boxes(const PrefixArgs& a, int c, int npages) {
    const int br = a.box_rows;
    int n = 0;
    for (int i = 0; i < kChunkTokens / br; ++i)
        if ((c * kChunkTokens + i * br) / a.page_size < npages) ++n;
    return n;
}

// The tokens of chunk c of KV head h (rows of the [page][kv_head][slot][dim]
// pool) into consecutive 128-byte rows at dst, as `boxes` boxes of box_rows
// rows (the later rows keep what they held: those tokens are masked).
__device__ __forceinline__ void load_chunk_rows(uint32_t dst, const CUtensorMap* map, const PrefixArgs& a,
                                                const int32_t* prow, int c, int h, int boxes, uint64_t* bar) {
    const int P = a.page_size, br = a.box_rows;
    for (int i = 0; i < boxes; ++i) {
        const int tok0 = c * kChunkTokens + i * br;
        int32_t pid = prow[tok0 / P];
        // (the plan admits only chunks whose page ids are valid; the clamp
        // keeps a table changed behind its back inside the pool)
        if (pid < 0 || pid >= a.num_pages) pid = 0;
        const int32_t y = (pid * a.num_kv_heads + h) * P + (tok0 % P);
        tma_load_2d(dst + i * br * 128, map, 0, y, bar);
    }
}

}  // namespace

// (at most 96 registers: 576 threads in one CTA, registers allocated per 4 warps)
__global__ void __maxnreg__(96)
prefix_attn_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                   const __grid_constant__ PrefixArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem0 = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int half = warp / kPfxHalfWarps;
    const int lwarp = warp - half * kPfxHalfWarps;            // warp within the half
    uint8_t* smem = smem0 + half * kPfxHalfBytes;
    uint64_t* full_k = reinterpret_cast<uint64_t*>(smem + kPfxBarOff);
    uint64_t* empty_k = full_k + 1;
    uint64_t* full_v = full_k + 2;
    uint64_t* empty_v = full_k + 3;
    uint64_t* mma_bar = full_k + 4;
    // (shared by both halves: in the first half's region)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem0 + kPfxBarOff + 40);
    volatile int* failed = reinterpret_cast<volatile int*>(smem0 + kPfxBarOff + 44);
    // exchange between the two threads of a row: maxima, then l and lr
    float* s_xmax = reinterpret_cast<float*>(smem + kPfxXOff);   // [256]
    float* s_xl = s_xmax + kPfxRowThreads;                       // [256]
    float* s_xlr = s_xl + kPfxRowThreads;                        // [256]

    launch_dependents();
    if (tid == 0) {
        for (int hf = 0; hf < 2; ++hf) {
            uint64_t* fb = reinterpret_cast<uint64_t*>(smem0 + hf * kPfxHalfBytes + kPfxBarOff);
            mbar_init(fb, 1);                   // K full
            mbar_init(fb + 1, kPfxRowWarps);    // K empty
            mbar_init(fb + 2, 1);               // V full
            mbar_init(fb + 3, kPfxRowWarps);    // V empty
            mbar_init(fb + 4, 1);               // tensor-core commits
        }
        *failed = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_slot), kPfxTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot + 256u * static_cast<uint32_t>(half);   // this half's columns

    // the plan and the abort flags come from the preceding kernels
    grid_dependency_wait();
    const int IPR = a.items_per_req;
    const int total = *a.num_tiles * IPR;
    const uint32_t base = smem_addr(smem);
    // A tile's steps: its shared chunks (read through the reference row), then
    // for each member the tile finishes (chunk_begin = all its chunks) the
    // chunks after its shared ones (read through its own row).
    auto n_chunks = [&](int bb) { return (a.seq_lens[bb] + kChunkTokens - 1) / kChunkTokens; };
    auto finished = [&](int bb) { return a.chunk_begin[bb] == n_chunks(bb); };

    if (lwarp == kPfxRowWarps) {
        // ================= producer =================
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
            uint32_t it = 0;
            auto load = [&](const int32_t* prow, int c, int p, int npages) {
                const int boxes = chunk_boxes(a, c, npages);
                const uint32_t bytes = 2u * boxes * a.box_rows * 128u;
                if (it > 0 && !gemv_wait(empty_k, (it - 1) & 1, failed, a.status)) return false;
                mbar_arrive_expect_tx(full_k, bytes);
                for (int hh = 0; hh < 2; ++hh)
                    load_chunk_rows(base + kPfxRawKOff + hh * (kPfxRawBytes / 2), &tmap_k, a, prow, c, 2 * p + hh,
                                    boxes, full_k);
                if (it > 0 && !gemv_wait(empty_v, (it - 1) & 1, failed, a.status)) return false;
                mbar_arrive_expect_tx(full_v, bytes);
                for (int hh = 0; hh < 2; ++hh)
                    load_chunk_rows(base + kPfxRawVOff + hh * (kPfxRawBytes / 2), &tmap_v, a, prow, c, 2 * p + hh,
                                    boxes, full_v);
                ++it;
                return true;
            };
            for (int ti = 2 * blockIdx.x + half; ti < total && !*failed; ti += 2 * gridDim.x) {
                const int t = ti / IPR, p = ti - t * IPR;
                const int32_t* prow = a.page_table + static_cast<int64_t>(a.tiles[4 * t]) * a.max_pages;
                const int b_first = a.tiles[4 * t + 1], nm = a.tiles[4 * t + 2], nch = a.tiles[4 * t + 3];
                for (int c = 0; c < nch; ++c)
                    if (!load(prow, c, p, INT_MAX)) break;
                for (int k = 0; k < nm; ++k) {
                    const int bb = b_first + k;
                    if (!finished(bb)) continue;
                    const int32_t* own = a.page_table + static_cast<int64_t>(bb) * a.max_pages;
                    const int npages = (a.seq_lens[bb] + a.page_size - 1) / a.page_size;
                    for (int c = a.pshare[bb]; c < n_chunks(bb); ++c)
                        if (!load(own, c, p, npages)) break;
                }
            }
        }
    } else {
        // ============ tile rows: warps 0-7, two threads per row ============
        // Row r = tensor-memory lane (warp w reaches lanes 32 (w mod 4) ..);
        // rows 0-63 hold the members' query heads of the pair's first KV
        // head, rows 64-127 of the second, so a warp's rows share a head.
        // The thread's half h2 picks half of the row's columns (S, P, O) and
        // of its dims (Q).
        // (a warp reaches the tensor-memory lanes 32 (w mod 4) .. of its
        // index w in the CTA)
        const int r = 32 * (warp & 3) + lane;
        const int h2 = lwarp >> 2;
        const int xi = h2 * kPfxRows + r;                    // this thread's exchange slot
        const bool issuer = lwarp == 0 && lane == 0;         // issues the half's tensor-core work
        const uint32_t tl = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
        const int G = a.group;
        const int hh = r >> 6;                               // KV head of the pair
        const int rr = r & 63;
        const int mrow = rr / G;                             // member
        const int g = rr - mrow * G;                         // query head in the group
        constexpr uint32_t idesc = mma_idesc_f16(128);
        constexpr uint32_t idesc_pv = mma_idesc_f16_bmn(128);   // V: N = dims contiguous
        uint32_t it = 0, mma_phase = 0;
        auto row_sync = [&]() { named_barrier_sync(1 + half, kPfxRowThreads); };
        auto mma_wait = [&]() {
            gemv_wait(mma_bar, mma_phase & 1, failed, a.status);
            ++mma_phase;
            tc_fence_after();
        };
        for (int ti = 2 * blockIdx.x + half; ti < total; ti += 2 * gridDim.x) {
            const int t = ti / IPR, p = ti - t * IPR;
            const int b_first = a.tiles[4 * t + 1], nm = a.tiles[4 * t + 2], nch = a.tiles[4 * t + 3];
            const bool real = mrow < nm && rr < a.members_per_tile * G;
            const int b = b_first + (real ? mrow : 0);
            const int ps = real ? a.pshare[b] : 0;
            const bool fin = real && finished(b);
            const bool dead = real && a.abort != nullptr && a.abort[b] != 0;
            const int hq = (2 * p + hh) * G + g;             // query head in the request

            // ---- Q row -> f16 scaled by 2^shift (exact), K-major swizzled tile ----
            float qs = 0.f;
            {
                uint4 w[8];
                const uint4* src = reinterpret_cast<const uint4*>(
                    a.q + (static_cast<int64_t>(b) * a.num_q_heads + hq) * kPfxD + 64 * h2);
#pragma unroll
                for (int j = 0; j < 8; ++j) w[j] = real ? src[j] : make_uint4(0u, 0u, 0u, 0u);
                float amax = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t x[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        amax = fmaxf(amax, fabsf(bf16_bits_to_f32(x[i] & 0xFFFFu)));
                        amax = fmaxf(amax, fabsf(bf16_bits_to_f32(x[i] >> 16)));
                    }
                }
                s_xmax[xi] = amax;
                row_sync();
                amax = fmaxf(s_xmax[r], s_xmax[r + kPfxRows]);
                // 2^shift brings amax into [128, 256) (see the split-K kernel)
                int shift = 0;
                if (amax > 0.f && isfinite(amax)) {
                    const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 126;
                    shift = min(60, max(-126, 8 - e));
                }
                const float up = __uint_as_float(static_cast<uint32_t>(shift + 127) << 23);
                qs = a.qk_scale * __uint_as_float(static_cast<uint32_t>(127 - shift) << 23);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t x[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
                    uint32_t h[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        h[i] = pack_f16x2(bf16_bits_to_f32(x[i] & 0xFFFFu) * up,
                                          bf16_bits_to_f32(x[i] >> 16) * up);
                    // dims 64 h2 + 8j .. + 7: atom h2, chunk j
                    sts128(base + kPfxQOff + h2 * kPfxAtom + atom_off(r, j), h[0], h[1], h[2], h[3]);
                }
            }
            fence_proxy_async_smem();
            row_sync();

            float m_run = kPfxNegInf, l_sum = 0.f, lr_sum = 0.f;
            // The tile's steps: shared chunks c < nch (member k = -1), then the
            // own chunks of each member the tile finishes.  Per step, `act`
            // says whether this row attends to the chunk, `valid` how many of
            // its 64 tokens exist (the others are masked, their V rows zero).
            int c = 0, cend = nch, k_mem = -1, len_k = 0;
            for (int step = 0;; ++step) {
                if (c >= cend) {
                    do {
                        ++k_mem;
                    } while (k_mem < nm && !finished(b_first + k_mem));
                    if (k_mem >= nm) break;
                    c = a.pshare[b_first + k_mem];
                    cend = n_chunks(b_first + k_mem);
                    len_k = a.seq_lens[b_first + k_mem];
                }
                const bool act = real && !dead && (k_mem < 0 ? c < ps : mrow == k_mem);
                const int valid = k_mem < 0 ? kChunkTokens : min(kChunkTokens, len_k - c * kChunkTokens);
                // ---- K: row r = token r mod 64 of head r / 64; dims 64 h2 .. ----
                gemv_wait(full_k, it & 1, failed, a.status);
                {
                    const uint32_t src = base + kPfxRawKOff + r * 128;
                    const uint32_t at = base + kPfxKVOff + h2 * kPfxAtom;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const uint32_t j = static_cast<uint32_t>(4 * h2 + jj);   // raw dims 16j .. 16j + 15
                        const uint4 x = lds128(src + ((j ^ (r & 7u)) << 4));
                        uint32_t f[8];
                        e4m3x4_to_f16x2x2(x.x, f[0], f[1]);
                        e4m3x4_to_f16x2x2(x.y, f[2], f[3]);
                        e4m3x4_to_f16x2x2(x.z, f[4], f[5]);
                        e4m3x4_to_f16x2x2(x.w, f[6], f[7]);
                        sts128(at + atom_off(r, (2 * jj) & 7), f[0], f[1], f[2], f[3]);
                        sts128(at + atom_off(r, (2 * jj + 1) & 7), f[4], f[5], f[6], f[7]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_k);
                fence_proxy_async_smem();
                tc_fence_before();
                row_sync();
                if (issuer) {
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t off = (k >> 2) * kPfxAtom + 32 * (k & 3);
                        tc_mma_ss(tmem, sw128_kmajor_desc(base + kPfxQOff + off),
                                  sw128_kmajor_desc(base + kPfxKVOff + off), idesc, k > 0 ? 1u : 0u);
                    }
                    tc_commit(mma_bar);
                }
                mma_wait();   // S is in tensor memory; the converted tile is free

                // ---- V: row r = token r mod 64 of head r / 64; dims 64 h2 .. ----
                // (token rows of 64-dim blocks, as the MN-major operand of
                // O += P V: no transpose; the rows of missing tokens are zero)
                gemv_wait(full_v, it & 1, failed, a.status);
                {
                    const bool zero = rr >= valid;
                    const uint32_t src = base + kPfxRawVOff + r * 128;
                    const uint32_t at = base + kPfxKVOff + h2 * kPfxAtom;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const uint32_t j = static_cast<uint32_t>(4 * h2 + jj);   // raw dims 16 j .. 16 j + 15
                        uint4 x = lds128(src + ((j ^ (r & 7u)) << 4));
                        if (zero) x = make_uint4(0u, 0u, 0u, 0u);
                        uint32_t f[8];
                        e4m3x4_to_f16x2x2(x.x, f[0], f[1]);
                        e4m3x4_to_f16x2x2(x.y, f[2], f[3]);
                        e4m3x4_to_f16x2x2(x.z, f[4], f[5]);
                        e4m3x4_to_f16x2x2(x.w, f[6], f[7]);
                        sts128(at + atom_off(r, (2 * jj) & 7), f[0], f[1], f[2], f[3]);
                        sts128(at + atom_off(r, (2 * jj + 1) & 7), f[4], f[5], f[6], f[7]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_v);
                fence_proxy_async_smem();

                // ---- online softmax; P (f16) over S in tensor memory ----
                // this thread: tokens 32 h2 .. 32 h2 + 31 of the row's head
                {
                    float sc[32];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        uint32_t v[16];
                        tmem_ld16(tl + static_cast<uint32_t>(hh * 64 + 32 * h2 + 16 * q), v);
                        tmem_wait_ld(v);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            sc[16 * q + i] = (32 * h2 + 16 * q + i < valid) ? __uint_as_float(v[i]) * qs : kPfxNegInf;
                    }
                    float m4[4] = {sc[0], sc[1], sc[2], sc[3]};
#pragma unroll
                    for (int i = 4; i < 32; ++i) m4[i & 3] = fmaxf(m4[i & 3], sc[i]);
                    s_xmax[xi] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                    row_sync();
                    const float mx = fmaxf(s_xmax[r], s_xmax[r + kPfxRows]);
                    // the running maximum grows past the threshold: rescale l, lr and
                    // this thread's half of the row of O (empty before the row's
                    // first chunk, which resets it)
                    const bool need = act && mx > m_run + kPfxLog2RescaleThreshold;
                    const float alpha = (need && m_run != kPfxNegInf) ? exp2f(m_run - mx) : 1.f;
                    if (need) {
                        l_sum *= alpha;
                        lr_sum *= alpha;
                        m_run = mx;
                    }
                    if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint32_t v[16];
                            const uint32_t col = tl + kPfxOCol + 64 * h2 + 16 * q;
                            tmem_ld16(col, v);
                            tmem_wait_ld(v);
#pragma unroll
                            for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
                            tmem_st16(col, v);
                        }
                    }
                    // lr sums the weights as rounded to f16 for the product
                    // (read as binary32 times 2^-112, the sum scaled once)
                    uint32_t pw[16];
                    float ls[2] = {0.f, 0.f}, lrs[2] = {0.f, 0.f};
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float p0 = ex2_approx(sc[2 * i] - m_run), p1 = ex2_approx(sc[2 * i + 1] - m_run);
                        pw[i] = act ? pack_f16x2(p0, p1) : 0u;
                        ls[i & 1] += act ? p0 + p1 : 0.f;
                        float r0, r1;
                        f16x2_nonneg_scaled(pw[i], r0, r1);
                        lrs[i & 1] += r0 + r1;
                    }
                    l_sum += ls[0] + ls[1];
                    lr_sum += (lrs[0] + lrs[1]) * 0x1p112f;
                    // P columns 0-31: tokens of head 0, 32-63: head 1; this
                    // thread writes its 16 columns of its head and zeros in the
                    // matching columns of the other head
                    tmem_st16(tl + static_cast<uint32_t>(32 * hh + 16 * h2), pw);
                    tmem_st16_zero(tl + static_cast<uint32_t>(32 * (1 - hh) + 16 * h2));
                    tmem_wait_st();
                }
                tc_fence_before();
                row_sync();
                if (issuer) {
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {   // tokens 16 k .. 16 k + 15: two 8-row atoms
                        tc_mma_ts(tmem + kPfxOCol, tmem + 8 * k,
                                  sw128_mnmajor_desc(base + kPfxKVOff + 2048 * k, kPfxAtom), idesc_pv,
                                  (step > 0 || k > 0) ? 1u : 0u);
                    }
                    tc_commit(mma_bar);
                }
                mma_wait();   // O updated; P, S and the converted tile are free
                ++c;
                ++it;
            }

            // ---- this row: final output (a member the tile finishes) or the
            // record (m, l, lr, 0) and O with the V scale applied ----
            // (every lane reads its half of the O row: the loads are warp-wide)
            {
                s_xl[xi] = l_sum;
                s_xlr[xi] = lr_sum;
                row_sync();
                const float l_tot = s_xl[r] + s_xl[r + kPfxRows];
                const float lr_tot = s_xlr[r] + s_xlr[r + kPfxRows];
                const int64_t item = static_cast<int64_t>(b) * IPR + p;
                const int IQ = 2 * G;
                const int hi = hh * G + g;                    // head within the item
                const bool live = real && !dead;
                const int64_t orow = static_cast<int64_t>(b) * a.num_q_heads + hq;
                const float k_out = live ? a.v_scale / lr_tot : 0.f;
                const float vs = live ? a.v_scale : 0.f;
                float4* o = reinterpret_cast<float4*>(a.pfx_o + (item * IQ + hi) * kPfxD + 64 * h2);
                uint32_t* dst = reinterpret_cast<uint32_t*>(a.out + orow * kPfxD + 64 * h2);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t v[16];
                    tmem_ld16(tl + kPfxOCol + 64 * h2 + 16 * q, v);
                    tmem_wait_ld(v);
                    if (fin) {
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * k_out, __uint_as_float(v[2 * i + 1]) * k_out);
#pragma unroll
                        for (int i = 0; i < 8; ++i) dst[8 * q + i] = pk[i];
                    } else if (real) {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            o[4 * q + i] = make_float4(__uint_as_float(v[4 * i]) * vs, __uint_as_float(v[4 * i + 1]) * vs,
                                                       __uint_as_float(v[4 * i + 2]) * vs,
                                                       __uint_as_float(v[4 * i + 3]) * vs);
                    }
                }
                if (h2 == 0 && real) {
                    if (fin) {
                        a.lse[orow] = live ? (m_run + log2f(l_tot)) * kPfxLn2 : kPfxNegInf;
                    } else {
                        float4* ml = reinterpret_cast<float4*>(a.pfx_ml + (item * IQ + hi) * 4);
                        *ml = live ? make_float4(m_run, l_tot, lr_tot, 0.f) : make_float4(kPfxNegInf, -1.f, -1.f, 0.f);
                    }
                }
                tc_fence_before();
                row_sync();
            }
            // the next tile rewrites Q, whose last reader (the final S product)
            // has completed, O, read above by every row, and the exchange
            // arrays, read above (the next writes follow another barrier)
        }
    }

    // every MMA of this CTA has completed (waited above): free the columns
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(*tmem_slot, kPfxTmemCols);
    }
}

// ---------------------------------------------------------------------------
// launches
// ---------------------------------------------------------------------------
size_t prefix_attn_smem_bytes() { return kPfxSmemBytes; }

cudaError_t prefix_set_smem_attr() {
    cudaError_t e =
        cudaFuncSetAttribute(prefix_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPfxSmemBytes);
    if (e != cudaSuccess) return e;
    // all of the SM's on-chip memory as shared memory: two CTAs per SM
    return cudaFuncSetAttribute(prefix_attn_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                cudaSharedmemCarveoutMaxShared);
}

cudaError_t prefix_occupancy(int* blocks_per_sm) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, prefix_attn_kernel, kPfxThreads,
                                                         kPfxSmemBytes);
}

cudaError_t prefix_attributes(int* regs, int* local_bytes, int* max_threads) {
    cudaFuncAttributes at;
    cudaError_t e = cudaFuncGetAttributes(&at, prefix_attn_kernel);
    *regs = at.numRegs;
    *local_bytes = static_cast<int>(at.localSizeBytes);
    *max_threads = at.maxThreadsPerBlock;
    return e;
}

cudaError_t launch_prefix_plan(cudaStream_t stream, const PrefixArgs& args) {
    const dim3 warps_grid((args.batch + 7) / 8);
    {
        PdlLaunch l(warps_grid, dim3(256), 0, stream);
        cudaError_t e = cudaLaunchKernelEx(&l.cfg, prefix_link_kernel, args);
        if (e != cudaSuccess) return e;
    }
    {
        PdlLaunch l(dim3(1), dim3(kPfxPlanThreads), 0, stream);
        cudaError_t e = cudaLaunchKernelEx(&l.cfg, prefix_group_kernel, args);
        if (e != cudaSuccess) return e;
    }
    {
        PdlLaunch l(warps_grid, dim3(256), 0, stream);
        cudaError_t e = cudaLaunchKernelEx(&l.cfg, prefix_share_kernel, args);
        if (e != cudaSuccess) return e;
    }
    PdlLaunch l(dim3(1), dim3(kPfxPlanThreads), 0, stream);
    return cudaLaunchKernelEx(&l.cfg, prefix_tile_kernel, args);
}

cudaError_t launch_prefix_attn(int grid, cudaStream_t stream, const CUtensorMap& tmap_k,
                               const CUtensorMap& tmap_v, const PrefixArgs& args) {
    PdlLaunch l(dim3(grid), dim3(kPfxThreads), kPfxSmemBytes, stream);
    return cudaLaunchKernelEx(&l.cfg, prefix_attn_kernel, tmap_k, tmap_v, args);
}

}  // namespace pkv
