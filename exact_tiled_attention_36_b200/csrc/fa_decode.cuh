// fa_decode.cuh: split-KV attention for a few query tokens per sequence against a
// long key/value cache (decode, speculative decode) on sm_100a.
//
// With Nq small the forward's 128-row query tiles would be nearly empty and every
// query head would read its KV head again. Here the rows of one work item are the
// queries of a whole KV-head group: R = (Hq / Hkv) * Nq <= 128 rows, one tile,
// so every K/V tile is read from HBM once per (sequence, KV head). The item walks
// its key tiles with the online softmax of the forward ("FlashAttention/zh",
// section "FlashAttention algorithm": running max m, normaliser l, rescale of the
// partial output, O / l and L = m + log l).
//
// Split over the keys (stream-K): the items' key tiles, laid end to end in item
// order (item = (sequence, KV head)), form one sequence of T tiles, and CTA c of G
// takes tiles [floor(c T / G), floor((c + 1) T / G)): every CTA gets the same
// number of tiles up to one, whatever the sequences' lengths. Where a CTA's range
// crosses an item boundary it runs one segment per item. Each segment leaves a
// partial output O_s (normalised by its own sum) and log-sum-exp L_s in slot c + i
// (i the item; unique, because a CTA whose range reaches item i + 1 ends before
// CTA c + 1 starts), and fa_decode_combine merges the segments of an item with
//     L = log sum_s exp(L_s),   O = sum_s exp(L_s - L) O_s,
// the rescaling step of the online softmax applied across segments (exact).
//
// Row layout: query row r = t g + h (token t, head h of the group of g) holds
// TMEM lane lane(r). When the group's heads split into nb = 2 or 4 blocks of
// gh = g / nb heads with gh Nq <= 32, block k sits in lanes 32 k .. 32 k + 31 (one
// TMA box per block) so that the rows spread over the four warps of the softmax
// warpgroup, and with them the exponentials over the four SM sub-partitions;
// otherwise (nb = 1) the rows fill lanes 0 .. R-1. Lanes that hold no row read a
// zero row of Q; their results are never used.
//
// Warp roles (256 threads): warp 0 TMA producer (Q per segment, K/V through an
// mbarrier ring), warp 1 TMEM allocation and the single MMA thread, warps 4-7 the
// softmax (thread l owns TMEM lane l; warps without a row stay out), warps 2-3
// idle. TMEM: S_0 / P_0 [0,128), S_1 / P_1 [128,256), O [256,256+d). The MMA
// thread issues S for key tile g + 2 right after O += P V of tile g, so the
// softmax of one tile overlaps the products of the next.
//
// Sequences of their own length (cache_seqlens) and a paged cache (block_table)
// are template options; rows of the last tile past the sequence's length are
// masked in S and zeroed in the V tile (the cache may hold anything there).
#pragma once

#include "sm100.cuh"

namespace fa {

struct DecodeArgs {
    void* o;               // [B, Nq, Hq, d] 16-bit (written by the combine)
    float* lse;            // [B, Hq, Nq]
    float* o_part;         // [slots, R, d] fp32 partial outputs
    float* lse_part;       // [slots, R]
    long long* meta;       // [0] = T, [1 + i] = first tile of item i (sequence lengths given)
    const int* seqlens;    // [B] or null (every sequence has Nk keys)
    const int* block_table;  // paged: [B, max_pages]
    int B, Hq, Hkv, group, Nq, Nk, R;
    int cap;               // keys a sequence can hold (Nk, or max_pages * page_size)
    int page_size, max_pages, page_box;  // paged: rows per page, pages per sequence, rows per TMA box
    int nb, gh;            // row layout: head blocks and heads per block
    int pair, rg, r8;      // narrow, d = 64: items are pairs of KV heads (see fa_decode_narrow_kernel);
                           // rg rows per KV head, the second head's rows from tile row r8
    int G;                 // CTAs of the split kernel
    float scale_log2;
    int* err;
};

constexpr int kDecThreads = 256;

template <int D>
struct DecCfg {
    static constexpr int kSlabs = D / 64;
    static constexpr int kSlabBytes = 128 * 128;
    static constexpr int kTileBytes = kSlabs * kSlabBytes;
    static constexpr int kStages = (D == 128) ? 3 : 4;
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + kTileBytes;
    static constexpr int kVOff = kKOff + kStages * kTileBytes;
    static constexpr int kBarOff = kVOff + kStages * kTileBytes;
    static constexpr int kNumBars = 2 + 4 * kStages + 2 + 2 + 5;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 128;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0, kColO = 256;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Query row held by TMEM lane l (-1: none).
__device__ __forceinline__ int dec_row(const DecodeArgs& a, int l) {
    const int blk = a.nb > 1 ? (l >> 5) : 0;
    const int loc = l - 32 * blk;
    if (blk >= a.nb || loc >= a.gh * a.Nq) return -1;
    return (loc / a.gh) * a.group + blk * a.gh + loc % a.gh;
}

// Softmax warps that hold at least one row.
__device__ __forceinline__ int dec_active_warps(const DecodeArgs& a) {
    return a.nb > 1 ? a.nb : (a.R + 31) / 32;
}

// The split balances cost, not tiles: an item of ntk > 0 key tiles costs
// ntk + kDecItemCost units, the first kDecItemCost standing for a segment's fixed
// work (loading Q, the first products, the epilogue). Otherwise a CTA whose share
// starts many short items would take longer than one with the same tiles of a
// single item.
constexpr int kDecItemCost = 2;

// One item (sequence b, KV head hk): its keys, and the first unit of its cost in the
// sequence of T units (its tiles are units P + kDecItemCost ..).
struct DecItem {
    int b, hk, len, ntk, cost;
    long long P;
};

template <bool SEQLENS>
__device__ __forceinline__ int dec_len(const DecodeArgs& a, int b) {
    if constexpr (SEQLENS) return min(max(a.seqlens[b], 0), a.cap);
    return a.Nk;
}

template <bool SEQLENS>
__device__ __forceinline__ DecItem dec_item(const DecodeArgs& a, int b, int hk, long long P) {
    DecItem it;
    it.b = b;
    it.hk = hk;
    it.P = P;
    it.len = dec_len<SEQLENS>(a, b);
    it.ntk = (it.len + 127) / 128;
    it.cost = it.ntk > 0 ? it.ntk + kDecItemCost : 0;
    return it;
}

// The key tiles [j0, j0 + n) of item `it` in the cost range [s_lo, s_hi) of a CTA
// (false: none).
__device__ __forceinline__ bool dec_segment(long long s_lo, long long s_hi, const DecItem& it, int& j0, int& n) {
    const long long r0 = it.P + kDecItemCost;  // the unit of the item's first tile
    const long long lo = max(s_lo, r0), hi = min(s_hi, it.P + it.cost);
    if (lo >= hi) return false;
    j0 = static_cast<int>(lo - r0);
    n = static_cast<int>(hi - lo);
    return true;
}

// The item after `it`; past the last one P = T (the walk ends there).
template <bool SEQLENS>
__device__ __forceinline__ DecItem dec_next(const DecodeArgs& a, const DecItem& it, long long T) {
    if (it.hk + 1 < a.Hkv) return dec_item<SEQLENS>(a, it.b, it.hk + 1, it.P + it.cost);
    if (it.b + 1 < a.B) return dec_item<SEQLENS>(a, it.b + 1, 0, it.P + it.cost);
    DecItem e = it;
    e.P = T;
    e.ntk = e.cost = 0;
    return e;
}

// CTA whose tile range holds tile t: the largest c with floor(c T / G) <= t.
__device__ __forceinline__ int dec_cta_of(long long t, long long T, int G) {
    return static_cast<int>(((t + 1) * G - 1) / T);
}

__device__ __forceinline__ long long dec_split(int c, long long T, int G) { return (static_cast<long long>(c) * T) / G; }


// The CTA's tile range [s_lo, s_hi) of the T tiles and the item holding s_lo.
struct DecRange {
    long long T, s_lo, s_hi;
    DecItem first;
};

// Called by every thread of the CTA (it synchronises the CTA when sequence lengths
// are given: every CTA then sums the per-sequence tile counts itself, a block
// reduction, and finds the sequence holding its first tile, a block scan). Returns
// false, for every thread, when the CTA has no tile. Uses 112 bytes at `misc + 8`.
template <bool SEQLENS>
__device__ __forceinline__ bool dec_locate(const DecodeArgs& args, uint8_t* misc, DecRange& rg) {
    const int G = args.G;
    const int cta = static_cast<int>(blockIdx.x);
    const int tid = static_cast<int>(threadIdx.x);
    const int warp = warp_id();
    const int lane = lane_id();
    constexpr int kWarps = kDecThreads / 32;
    long long T, s_lo, s_hi;
    int b0;
    long long P0;  // first tile of sequence b0 (its KV head 0)
    if constexpr (SEQLENS) {
        int* found = reinterpret_cast<int*>(misc + 8);
        int* sh_b0 = reinterpret_cast<int*>(misc + 24);
        long long* sh_P0 = reinterpret_cast<long long*>(misc + 32);
        long long* ws = reinterpret_cast<long long*>(misc + 48);  // [8] per-warp sums
        auto tiles_of = [&](int b) -> long long {  // cost units of sequence b (all its KV heads)
            if (b >= args.B) return 0;
            const int ntk = (dec_len<true>(args, b) + 127) / 128;
            return ntk > 0 ? static_cast<long long>(args.Hkv) * (ntk + kDecItemCost) : 0;
        };
        long long v = 0;
        for (int b = tid; b < args.B; b += kDecThreads) v += tiles_of(b);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) ws[warp] = v;
        if (tid == 0) *found = 0;
        __syncthreads();
        T = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) T += ws[w];
        if (cta == 0 && tid == 0) args.meta[0] = T;
        s_lo = dec_split(cta, T, G);
        s_hi = dec_split(cta + 1, T, G);
        if (s_lo >= s_hi) return false;  // fewer tiles than CTAs (uniform)
        __syncthreads();                 // every thread has read ws
        long long run = 0;
        for (int base = 0; base < args.B; base += kDecThreads) {
            const int b = base + tid;
            const long long x = tiles_of(b);
            long long incl = x;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            if (lane == 31) ws[warp] = incl;
            __syncthreads();
            long long before = 0, total = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const long long y = ws[w];
                if (w < warp) before += y;
                total += y;
            }
            const long long excl = run + before + incl - x;
            if (x > 0 && excl <= s_lo && s_lo < excl + x) {  // one thread at most
                *sh_b0 = b;
                *sh_P0 = excl;
                *found = 1;
            }
            __syncthreads();
            if (*found) break;
            run += total;
        }
        if (!*found) return false;  // cannot happen: s_lo < T
        b0 = *sh_b0;
        P0 = *sh_P0;
    } else {
        const int ntk = (args.Nk + 127) / 128;
        const long long per_b = ntk > 0 ? static_cast<long long>(args.Hkv) * (ntk + kDecItemCost) : 0;
        T = per_b * args.B;
        s_lo = dec_split(cta, T, G);
        s_hi = dec_split(cta + 1, T, G);
        if (s_lo >= s_hi) return false;
        b0 = static_cast<int>(s_lo / per_b);
        P0 = b0 * per_b;
    }
    const int cost = (dec_len<SEQLENS>(args, b0) + 127) / 128 + kDecItemCost;  // of each KV head of b0
    const int hk = static_cast<int>((s_lo - P0) / cost);
    rg.T = T;
    rg.s_lo = s_lo;
    rg.s_hi = s_hi;
    rg.first = dec_item<SEQLENS>(args, b0, hk, P0 + static_cast<long long>(hk) * cost);
    return true;
}

// The TMA producer (one thread): per segment the group's query rows (nb boxes of
// gh heads x Nq tokens, box k at q_block_off * k within each 64-column slab of
// q_slab_bytes) into Q buffer nq % QB (q_tile_bytes apart), then every K and V tile
// of the segment through the S-stage rings. With two Q buffers the next segment's Q
// (and so its K and V) load while the current segment's products still read its Q.
// K and V tiles are 128 keys x d (16-bit), 64-column slabs of 16 KB.
template <int D, bool SEQLENS, bool PAGED, int S, int QB = 1>
__device__ __forceinline__ void dec_produce(const DecodeArgs& args, const DecRange& rg, const CUtensorMap* tm_q,
                                            const CUtensorMap* tm_k, const CUtensorMap* tm_v, uint8_t* sQ,
                                            int q_slab_bytes, int q_block_off, uint8_t* sK, uint8_t* sV,
                                            uint64_t* q_full, uint64_t* q_empty, uint64_t* k_full, uint64_t* k_empty,
                                            uint64_t* v_full, uint64_t* v_empty, const WaitCtx& wc,
                                            int q_tile_bytes = 0) {
    constexpr int kSlabs = D / 64;
    constexpr int kSlabBytes = 128 * 128;
    constexpr int kTileBytes = kSlabs * kSlabBytes;
    const int g = args.group;
    int gk = 0, nq = 0, k_issued = 0, v_issued = 0;
    bool ok = true;
    // Paged: the pages of one key tile (boxes of page_box rows; one page holds whole
    // boxes), read from the block table once per tile for both K and V, all reads in
    // flight together. Boxes past the sequence's end are not loaded (their rows are
    // masked, and zeroed in V).
    constexpr int kMaxBoxes = 8;  // 128 keys / 16-row pages
    int pages[kMaxBoxes];
    int boxes = 0;
    auto read_pages = [&](const DecItem& it, int kt) {
        if constexpr (PAGED) {
            const int pb = args.page_box;
            boxes = (min(128, it.len - kt * 128) + pb - 1) / pb;
            const int* bt = args.block_table + static_cast<size_t>(it.b) * args.max_pages;
#pragma unroll
            for (int x = 0; x < kMaxBoxes; ++x)
                pages[x] = x < boxes ? bt[(kt * 128 + x * pb) / args.page_size] : 0;
        }
    };
    // One K or V tile (key tile kt of item `it`) into ring buffer `dst`.
    auto load_kv = [&](uint8_t* dst, const CUtensorMap* m, uint64_t* bar, const DecItem& it, int kt) {
        if constexpr (!PAGED) {
            mbar_arrive_expect_tx(bar, kTileBytes);
#pragma unroll
            for (int s = 0; s < kSlabs; ++s) tma_load_4d(dst + s * kSlabBytes, m, bar, s * 64, it.hk, kt * 128, it.b);
        } else {
            const int pb = args.page_box;
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(boxes * pb * 128 * kSlabs));
#pragma unroll
            for (int x = 0; x < kMaxBoxes; ++x) {
                if (x >= boxes) break;
                const int key = kt * 128 + x * pb;
#pragma unroll
                for (int s = 0; s < kSlabs; ++s)
                    tma_load_4d(dst + s * kSlabBytes + x * pb * 128, m, bar, s * 64, it.hk, key % args.page_size,
                                pages[x]);
            }
        }
    };
    for (DecItem it = rg.first; ok && it.P < rg.s_hi; it = dec_next<SEQLENS>(args, it, rg.T)) {
        if (SEQLENS && it.cost > 0 && it.P >= rg.s_lo)  // the item starts in this CTA's range
            args.meta[1 + static_cast<size_t>(it.b) * args.Hkv + it.hk] = it.P;
        int j0, n;
        if (!dec_segment(rg.s_lo, rg.s_hi, it, j0, n)) continue;
        // Q of the group once the last S product of the segment that used this buffer
        // before has read it.
        const int qb = nq % QB;
        uint8_t* q_dst = sQ + qb * q_tile_bytes;
        if (!(ok = mbar_wait(&q_empty[qb], ((nq / QB) & 1) ^ 1u, wc, 80))) break;
        mbar_arrive_expect_tx(&q_full[qb],
                              static_cast<uint32_t>(args.pair ? 2 * 128 * args.rg : kSlabs * 128 * args.R));
        if (args.pair) {
            // KV heads 2 hk and 2 hk + 1 (64 columns each): the first group's rows in
            // columns 0..63 from row 0, the second's in columns 64..127 from row r8.
#pragma unroll
            for (int k = 0; k < 2; ++k)
                tma_load_4d(q_dst + k * q_slab_bytes + k * args.r8 * 128, tm_q, &q_full[qb], 0, (2 * it.hk + k) * g,
                            0, it.b);
        } else {
            for (int k = 0; k < args.nb; ++k)
#pragma unroll
                for (int s = 0; s < kSlabs; ++s)
                    tma_load_4d(q_dst + s * q_slab_bytes + k * q_block_off, tm_q, &q_full[qb], s * 64,
                                it.hk * g + k * args.gh, 0, it.b);
        }
        ++nq;
        for (int j = 0; j < n; ++j) {
            const int gg = gk + j, st = gg % S;
            const uint32_t ph = (gg / S) & 1;
            read_pages(it, j0 + j);
            if (!(ok = mbar_wait(&k_empty[st], ph ^ 1u, wc, 81))) break;
            load_kv(sK + st * kTileBytes, tm_k, &k_full[st], it, j0 + j);
            ++k_issued;
            if (!(ok = mbar_wait(&v_empty[st], ph ^ 1u, wc, 82))) break;
            load_kv(sV + st * kTileBytes, tm_v, &v_full[st], it, j0 + j);
            ++v_issued;
        }
        gk += n;
    }
    // Leave no load in flight: wait for the last one issued into every buffer.
    for (int qb = 0; qb < QB; ++qb) {
        const int uses = (nq + QB - 1 - qb) / QB;  // loads into Q buffer qb
        if (uses > 0) mbar_wait_drain(&q_full[qb], (uses - 1) & 1);
    }
    for (int st = 0; st < S; ++st) {
        if (k_issued > st) mbar_wait_drain(&k_full[st], ((st + S * ((k_issued - 1 - st) / S)) / S) & 1);
        if (v_issued > st) mbar_wait_drain(&v_full[st], ((st + S * ((v_issued - 1 - st) / S)) / S) & 1);
    }
}

// PAGED: k and v are page pools [num_pages, page_size, Hkv, d] addressed through
// block_table (requires SEQLENS). SEQLENS: sequence b has seqlens[b] keys (clamped
// to [0, cap]); else every sequence has Nk. causal (runtime): query t of a
// sequence of n keys sees keys 0 .. t + n - Nq (bottom-right alignment).
template <int D, bool BF16, bool SEQLENS, bool PAGED>
__global__ void __launch_bounds__(kDecThreads, 1)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const DecodeArgs args, const int causal) {
    static_assert(SEQLENS || !PAGED, "a paged cache needs the sequence lengths");
    using C = DecCfg<D>;
    constexpr int S = C::kStages;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (!smem_base_ok(smem, args.err)) return;
    // The merge kernel may be scheduled now; it waits for this grid before reading.
    asm volatile("griddepcontrol.launch_dependents;");
    const int cta = static_cast<int>(blockIdx.x);
    const int tid = static_cast<int>(threadIdx.x);
    const int warp = warp_id();
    const int lane = lane_id();
    uint8_t* misc = smem + C::kMiscOff;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(misc);
    int* abort_flag = reinterpret_cast<int*>(misc + 4);

    DecRange rg;
    if (!dec_locate<SEQLENS>(args, misc, rg)) return;  // no tile for this CTA
    const long long T = rg.T, s_lo = rg.s_lo, s_hi = rg.s_hi;
    const DecItem first = rg.first;

    uint8_t* sQ = smem + C::kQOff;
    uint8_t* sK = smem + C::kKOff;
    uint8_t* sV = smem + C::kVOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* q_full = bars;
    uint64_t* q_empty = bars + 1;  // the segment's last S product has read Q
    uint64_t* k_full = bars + 2;
    uint64_t* k_empty = k_full + S;
    uint64_t* v_full = k_empty + S;
    uint64_t* v_empty = v_full + S;
    uint64_t* s_full = v_empty + S;  // [2] S buffers
    uint64_t* p_full = s_full + 2;   // [2]
    uint64_t* pv_done = p_full + 2;  // one completion per O += P V
    uint64_t* o_ready = pv_done + 1;  // every product of the segment is complete
    uint64_t* o_free = o_ready + 1;   // the epilogue has read O
    uint64_t* mma_done = o_free + 1;
    uint64_t* sm_done = mma_done + 1;
    const int n_act = 32 * dec_active_warps(args);  // softmax threads that take part

    // Lanes that hold no query row read zeros (loaded rows are the same for every
    // segment, so this is done once).
    for (int i = tid; i < C::kTileBytes / 16; i += kDecThreads) {
        const int row = (i % (C::kSlabBytes / 16)) / 8;
        if (dec_row(args, row) < 0) reinterpret_cast<uint4*>(sQ)[i] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    if (tid == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < S; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], n_act);
        }
        mbar_init(pv_done, 1);
        mbar_init(o_ready, 1);
        mbar_init(o_free, n_act);
        mbar_init(mma_done, 1);
        mbar_init(sm_done, n_act);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_holder);
    const WaitCtx wc{abort_flag, args.err};
    const int g = args.group;

    if (warp == 0) {
        if (lane == 0)
            dec_produce<D, SEQLENS, PAGED, S>(args, rg, &tm_q, &tm_k, &tm_v, sQ, C::kSlabBytes,
                                              args.nb > 1 ? 4096 : 0, sK, sV, q_full, q_empty, k_full, k_empty,
                                              v_full, v_empty, wc);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_qk = idesc_f16(128, 128, BF16, false, false);
            constexpr uint32_t id_pv = idesc_f16(128, D, BF16, false, true);
            const uint32_t q_addr = smem_u32(sQ);
            // S into buffer gg % 2 from the K tile of ring index gg.
            auto issue_s = [&](int gg) {
                const uint32_t k_addr = smem_u32(sK + (gg % S) * C::kTileBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kSlabBytes + (kk & 3) * 32;
                    mma_ss(tmem + C::kColS + 128 * (gg & 1), sdesc_sw128(q_addr + off, 16, 1024),
                           sdesc_sw128(k_addr + off, 16, 1024), id_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(&s_full[gg & 1]);
                tc_commit(&k_empty[gg % S]);
            };
            int gk = 0, nq = 0;
            bool ok = true;
            for (DecItem it = first; ok && it.P < s_hi; it = dec_next<SEQLENS>(args, it, T)) {
                int j0, n;
                if (!dec_segment(s_lo, s_hi, it, j0, n)) continue;
                if (!(ok = mbar_wait(q_full, nq & 1, wc, 83))) break;
                for (int j = 0; ok && j < min(n, 2); ++j) {
                    const int gg = gk + j;
                    if (!(ok = mbar_wait(&k_full[gg % S], (gg / S) & 1, wc, 84))) break;
                    tc_fence_after();
                    issue_s(gg);
                }
                if (!ok) break;
                if (n <= 2) tc_commit(q_empty);
                for (int j = 0; ok && j < n; ++j) {
                    const int gg = gk + j, st = gg % S;
                    if (!(ok = mbar_wait(&v_full[st], (gg / S) & 1, wc, 85))) break;
                    // O is overwritten by the segment's first P V: the previous segment's
                    // epilogue must have read it.
                    if (j == 0 && nq > 0 && !(ok = mbar_wait(o_free, (nq - 1) & 1, wc, 86))) break;
                    if (!(ok = mbar_wait(&p_full[gg & 1], (gg >> 1) & 1, wc, 87))) break;
                    tc_fence_after();
                    const uint32_t v_addr = smem_u32(sV + st * C::kTileBytes);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(tmem + C::kColO, tmem + C::kColS + 128 * (gg & 1) + kk * 8,
                               sdesc_sw128(v_addr + kk * 2048, C::kSlabBytes, 1024), id_pv,
                               (j > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(pv_done);
                    tc_commit(&v_empty[st]);
                    // S of tile gg + 2 into the columns P was just read from: one thread's
                    // tcgen05.mma operations execute in issue order.
                    if (j + 2 < n) {
                        if (!(ok = mbar_wait(&k_full[(gg + 2) % S], ((gg + 2) / S) & 1, wc, 88))) break;
                        tc_fence_after();
                        issue_s(gg + 2);
                        if (j + 3 == n) tc_commit(q_empty);
                    }
                }
                tc_commit(o_ready);
                gk += n;
                ++nq;
            }
            tc_commit(mma_done);
            mbar_wait_drain(mma_done, 0);
            const uint32_t a = smem_u32(sm_done);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < 4000000000ull) {
            }
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    } else if (warp >= 4 && (warp - 4) * 32 < n_act) {
        // ------------------------------------------------------------ softmax / epilogue
        const int w4 = warp - 4;
        const int l_idx = w4 * 32 + lane;  // TMEM lane, index among the active threads
        const int r = dec_row(args, l_idx);
        const int t = r >= 0 ? r / g : 0;  // query token of the row
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(w4 * 32) << 16);
        const uint32_t o_addr = lane_base + C::kColO;
        const float sl2 = args.scale_log2;
        int gk = 0, nq = 0;
        bool ok = true;
        for (DecItem it = first; ok && it.P < s_hi; it = dec_next<SEQLENS>(args, it, T)) {
            int j0, n;
            if (!dec_segment(s_lo, s_hi, it, j0, n)) continue;
            // This row's keys [0, key_hi), relative to the segment's first key.
            int key_hi = it.len;
            if (causal) key_hi = min(it.len, t + it.len - args.Nq + 1);
            const int rel_hi = key_hi - j0 * 128;
            float m = -INFINITY, l = 0.f, lr = 0.f;
            for (int j = 0; j < n; ++j) {
                const int gg = gk + j;
                ok = warp_all(mbar_wait(&s_full[gg & 1], (gg >> 1) & 1, wc, 89));
                if (!ok) break;
                tc_fence_after();
                const uint32_t s_addr = lane_base + C::kColS + 128 * (gg & 1);
                const int lim = rel_hi - j * 128;  // columns >= lim are masked
                const bool need_mask = __any_sync(0xffffffffu, lim < 128);
                uint32_t sv[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + 32 * c, sv[c]);
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld_wait(sv[c]);
                if (need_mask) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c >= lim) sv[c >> 5][c & 31] = __float_as_uint(-INFINITY);
                }
                float mxp[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mxp[i] = -INFINITY;
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    mxp[i & 7] = fmax3(mxp[i & 7], __uint_as_float(sv[(2 * i) >> 5][(2 * i) & 31]),
                                       __uint_as_float(sv[(2 * i + 1) >> 5][(2 * i + 1) & 31]));
                const float mx = fmax3(fmax3(mxp[0], mxp[1], mxp[2]), fmax3(mxp[3], mxp[4], mxp[5]),
                                       fmaxf(mxp[6], mxp[7]));
                const float m_new = fmaxf(m, mx * sl2);
                float alpha = 1.f;
                bool resc = false;
                if (m_new > m + kRescaleThreshold) {
                    if (m != -INFINITY) {
                        alpha = ex2_approx(m - m_new);
                        resc = true;
                    }
                    m = m_new;
                }
                const float neg_m = (m == -INFINITY) ? 0.f : -m;
                const uint64_t c2 = f2_pack(sl2, sl2), m2 = f2_pack(neg_m, neg_m);
                uint64_t rs2[4] = {0, 0, 0, 0}, rsr2[4] = {0, 0, 0, 0};
                uint32_t pk[2][32];
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    const uint64_t x = f2_pack(__uint_as_float(sv[(2 * i) >> 5][(2 * i) & 31]),
                                               __uint_as_float(sv[(2 * i + 1) >> 5][(2 * i + 1) & 31]));
                    float y0, y1;
                    f2_unpack(f2_fma(x, c2, m2), y0, y1);
                    const float p0 = ex2_approx(y0);
                    const float p1 = ex2_approx(y1);
                    rs2[i & 3] = f2_add(rs2[i & 3], f2_pack(p0, p1));
                    const uint32_t u = pack2<BF16>(p0, p1);
                    rsr2[i & 3] = f2_add(rsr2[i & 3], f2_pack(unpack_lo<BF16>(u), unpack_hi<BF16>(u)));
                    pk[i >> 5][i & 31] = u;
                }
                tmem_st32(s_addr + 0, pk[0]);
                tmem_st32(s_addr + 32, pk[1]);
                l = l * alpha + f2_sum(f2_add(f2_add(rs2[0], rs2[1]), f2_add(rs2[2], rs2[3])));
                lr = lr * alpha + f2_sum(f2_add(f2_add(rsr2[0], rsr2[1]), f2_add(rsr2[2], rsr2[3])));
                // Rescale O once the previous tile's P V is complete (S of this tile only
                // guarantees the one before that).
                if (j > 0 && __any_sync(0xffffffffu, resc)) {
                    ok = warp_all(mbar_wait(pv_done, (gg - 1) & 1, wc, 90));
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t ov[32];
                        tmem_ld32(o_addr + c0, ov);
                        tmem_ld_wait(ov);
#pragma unroll
                        for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                        tmem_st32(o_addr + c0, ov);
                    }
                }
                // The sequence's last tile: rows of V past its end may hold anything
                // (0 x NaN would reach O), so they are zeroed before P V reads them. V's
                // previous use of this buffer is complete (S of this tile is).
                if (SEQLENS && j0 + j == it.ntk - 1 && (it.len & 127) != 0) {
                    ok = warp_all(mbar_wait(&v_full[gg % S], (gg / S) & 1, wc, 91));
                    if (!ok) break;
                    const int v0 = it.len & 127;
                    const int per_slab = (128 - v0) * 8;
                    uint8_t* vt = sV + (gg % S) * C::kTileBytes;
                    for (int x = l_idx; x < per_slab * C::kSlabs; x += n_act) {
                        const int s = x / per_slab, rem = x % per_slab;
                        *reinterpret_cast<uint4*>(vt + s * C::kSlabBytes + (v0 + rem / 8) * 128 + (rem % 8) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&p_full[gg & 1]);
            }
            if (!ok) break;
            ok = warp_all(mbar_wait(o_ready, nq & 1, wc, 92));
            if (!ok) break;
            tc_fence_after();
            const int slot = cta + it.b * args.Hkv + it.hk;
            const float inv_l = (lr > 0.f) ? 1.f / lr : 0.f;
            float* dst = args.o_part + (static_cast<size_t>(slot) * args.R + (r >= 0 ? r : 0)) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t ov[32];
                tmem_ld32(o_addr + c0, ov);
                tmem_ld_wait(ov);
                if (r >= 0) {
                    float4* d4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        d4[i] = make_float4(__uint_as_float(ov[4 * i]) * inv_l, __uint_as_float(ov[4 * i + 1]) * inv_l,
                                            __uint_as_float(ov[4 * i + 2]) * inv_l,
                                            __uint_as_float(ov[4 * i + 3]) * inv_l);
                }
            }
            tc_fence_before();
            mbar_arrive(o_free);
            if (r >= 0) {
                float L = -INFINITY;
                if (l > 0.f) {
                    float lg;
                    asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(l));
                    L = (m + lg) * kLn2;
                }
                args.lse_part[static_cast<size_t>(slot) * args.R + r] = L;
            }
            gk += n;
            ++nq;
        }
        tc_fence_before();
        mbar_arrive(sm_done);
    }
}

// ------------------------------------------------------------------------ narrow
// The narrow kernel, for R = (Hq / Hkv) * Nq <= 32 rows (one generated token with
// up to 32 query heads per KV head, or a few speculative tokens): the products are
// taken with the operands swapped, so that keys, not query rows, run along the 128
// TMEM lanes and the tensor core's M = 128:
//     S^T = K Q^T       (M = 128 keys, N = RN >= R query rows, K = d)
//     O^T += V^T P^T    (M = d, N = RN, K = 128 keys)
// Thread l of the softmax warpgroup owns key l of the tile and takes R
// exponentials per tile (not 128), so the kernel streams K and V at the memory's
// pace. All threads use one reference max per row: a tile that raises some row's
// max by more than 2^8 over the reference (or the segment's first tile) takes the
// cross-warp reduction, sets the reference to the exact max and rescales the
// normalisers and O^T; other tiles need one vote and one meeting of the four warps.
// P goes through shared memory as the [RN x 128] (keys contiguous) B operand of the
// second product.
// d = 64 with an even number of KV heads and at most 16 rows per head (`pair`):
// an item is two adjacent KV heads, whose K and V rows form one contiguous 256-byte
// row (a 128-byte row per head would halve what HBM delivers), and the kernel runs
// as d = 128 with a block-diagonal Q: the first head's query rows hold their 64
// values in columns 0..63 (zeros in 64..127), the second head's rows, from tile
// row r8, in columns 64..127. Then S^T holds each row's scores against its own
// head, and O^T lanes 64 k .. 64 k + 63 hold head k's outputs. Other d = 64 cases
// keep M = 128 in the second product: its A operand's second 64 rows read the next
// 16 KB of shared memory (V stages come before K stages, so that stays inside the
// buffer) and land in TMEM lanes 64..127, which nothing reads.
// TMEM: S^T_b at [32 b, 32 b + RN) for the kNS buffers, then O^T (lane = d index).
template <int D, int RN>
struct DecNarrowCfg {
    static constexpr int kSlabs = D / 64;
    static constexpr int kKVSlab = 128 * 128;             // 128 keys x 64 columns
    static constexpr int kTileBytes = kSlabs * kKVSlab;
    // S^T buffers (and P buffers): the MMA thread issues S^T of tile j + kNS right
    // after P V of tile j, so the softmax has kNS tiles of slack over the products'
    // latency (which, not the exponentials, bounds a short tile).
    static constexpr int kNS = (D == 128) ? (RN == 16 ? 3 : 2) : 4;
    static constexpr int kStages = (D == 128) ? 3 : (RN == 16 ? 6 : 5);
    static constexpr int kQSlab = RN * 128;               // RN rows x 64 columns
    static constexpr int kQBytes = kSlabs * kQSlab;       // one Q buffer (two: one per segment parity)
    static constexpr int kPSlab = RN * 128;               // RN rows x 64 keys
    static constexpr int kPBytes = 2 * kPSlab;            // 128 keys
    static constexpr int kQOff = 0;
    static constexpr int kPOff = kQOff + 2 * kQBytes;      // kNS P buffers
    static constexpr int kVOff = kPOff + kNS * kPBytes;
    static constexpr int kKOff = kVOff + kStages * kTileBytes;
    static constexpr int kBarOff = kKOff + kStages * kTileBytes;
    static constexpr int kNumBars = 4 + 4 * kStages + 3 * kNS + 4 + 5;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kFlagOff = kMiscOff + 128;        // int [2][4]: a warp's rows need the exact max
    static constexpr int kRedOff = kFlagOff + 32;          // float [2][4][RN]: per-warp maxima
    static constexpr int kSumOff = kRedOff + 2 * 4 * RN * 4;  // float [4][RN][2]: per-warp sums
    static constexpr int kSmemBytes = kSumOff + 4 * RN * 2 * 4;
    static constexpr uint32_t kColO = 32 * kNS;
    static constexpr uint32_t kTmemCols = kColO + 32 <= 128 ? 128 : 256;
    static_assert(RN == 16 || RN == 32, "N of the swapped products");
    static_assert(kStages >= kNS, "a V buffer is reused only after the P V that read it");
    static_assert(kQOff % 1024 == 0 && kPOff % 1024 == 0 && kVOff % 1024 == 0 && kKOff % 1024 == 0, "alignment");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Byte offset of key `key` (0..127) of row r in a [RN x 128] 16-bit K-major tile
// with the 128-byte swizzle (two 64-key slabs of RN rows).
template <int RN>
__device__ __forceinline__ uint32_t dec_p_offset(int r, int key) {
    return static_cast<uint32_t>((key >> 6) * (RN * 128) + r * 128 + ((((key & 63) >> 3) ^ (r & 7)) << 4) +
                                 (key & 7) * 2);
}

template <int D, bool BF16, bool SEQLENS, bool PAGED, int RN>
__global__ void __launch_bounds__(kDecThreads, 1)
    fa_decode_narrow_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const DecodeArgs args, const int causal) {
    static_assert(SEQLENS || !PAGED, "a paged cache needs the sequence lengths");
    using C = DecNarrowCfg<D, RN>;
    constexpr int S = C::kStages;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (!smem_base_ok(smem, args.err)) return;
    // The merge kernel may be scheduled now; it waits for this grid before reading.
    asm volatile("griddepcontrol.launch_dependents;");
    const int cta = static_cast<int>(blockIdx.x);
    const int tid = static_cast<int>(threadIdx.x);
    const int warp = warp_id();
    const int lane = lane_id();
    uint8_t* misc = smem + C::kMiscOff;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(misc);
    int* abort_flag = reinterpret_cast<int*>(misc + 4);

    DecRange rg;
    if (!dec_locate<SEQLENS>(args, misc, rg)) return;  // no tile for this CTA

    uint8_t* sQ = smem + C::kQOff;
    uint8_t* sP = smem + C::kPOff;
    uint8_t* sK = smem + C::kKOff;
    uint8_t* sV = smem + C::kVOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* q_full = bars;       // [2] Q buffer of segment parity
    uint64_t* q_empty = bars + 2;  // [2]
    uint64_t* k_full = bars + 4;
    uint64_t* k_empty = k_full + S;
    uint64_t* v_full = k_empty + S;
    uint64_t* v_empty = v_full + S;
    constexpr int NS = C::kNS;
    uint64_t* s_full = v_empty + S;   // [NS] S^T buffer b holds tile gg (gg % NS == b)
    uint64_t* p_full = s_full + NS;   // [NS]
    uint64_t* pv_done = p_full + NS;  // [NS] P V of the tile in P buffer b complete
    uint64_t* o_ready = pv_done + NS;
    uint64_t* o_free = o_ready + 1;
    uint64_t* mma_done = o_free + 1;
    uint64_t* sm_done = mma_done + 1;

    // Rows of Q that no load writes are zeros: rows R .. RN-1, and with paired KV heads
    // everything outside the two groups' blocks (rows 0..rg-1 of columns 0..63, rows
    // r8..r8+rg-1 of columns 64..127), which makes Q block-diagonal.
    for (int i = tid; i < 2 * C::kQBytes / 16; i += kDecThreads) {
        const int row = (i % (C::kQSlab / 16)) / 8, slab = (i / (C::kQSlab / 16)) % C::kSlabs;
        const bool loaded = args.pair ? (row >= slab * args.r8 && row < slab * args.r8 + args.rg) : row < args.R;
        if (!loaded) reinterpret_cast<uint4*>(sQ)[i] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
        }
        for (int i = 0; i < S; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int i = 0; i < NS; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 128);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(o_ready, 1);
        mbar_init(o_free, 128);
        mbar_init(mma_done, 1);
        mbar_init(sm_done, 128);
        for (int i = 0; i < 5; ++i) mbar_init(sm_done + 1 + i, 4);  // softmax warps meeting: one arrival per warp
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_holder);
    const WaitCtx wc{abort_flag, args.err};

    if (warp == 0) {
        if (lane == 0)
            dec_produce<D, SEQLENS, PAGED, S, 2>(args, rg, &tm_q, &tm_k, &tm_v, sQ, C::kQSlab, 0, sK, sV, q_full,
                                                 q_empty, k_full, k_empty, v_full, v_empty, wc, C::kQBytes);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_f16(128, RN, BF16, false, false);
            constexpr uint32_t id_pv = idesc_f16(128, RN, BF16, true, false);
            uint32_t q_addr = smem_u32(sQ);  // the current segment's Q buffer
            // S^T into columns 32 (gg % NS) from the K tile of ring index gg.
            auto issue_s = [&](int gg) {
                const uint32_t k_addr = smem_u32(sK + (gg % S) * C::kTileBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t ko = (kk >> 2) * C::kKVSlab + (kk & 3) * 32;
                    const uint32_t qo = (kk >> 2) * C::kQSlab + (kk & 3) * 32;
                    mma_ss(tmem + 32 * (gg % NS), sdesc_sw128(k_addr + ko, 16, 1024),
                           sdesc_sw128(q_addr + qo, 16, 1024), id_s, kk > 0 ? 1u : 0u);
                }
                tc_commit(&s_full[gg % NS]);
                tc_commit(&k_empty[gg % S]);
            };
            int gk = 0, nq = 0;
            bool ok = true;
            for (DecItem it = rg.first; ok && it.P < rg.s_hi; it = dec_next<SEQLENS>(args, it, rg.T)) {
                int j0, n;
                if (!dec_segment(rg.s_lo, rg.s_hi, it, j0, n)) continue;
                const int qb = nq & 1;
                q_addr = smem_u32(sQ + qb * C::kQBytes);
                if (!(ok = mbar_wait(&q_full[qb], (nq >> 1) & 1, wc, 100))) break;
                for (int j = 0; ok && j < min(n, NS); ++j) {
                    const int gg = gk + j;
                    if (!(ok = mbar_wait(&k_full[gg % S], (gg / S) & 1, wc, 101))) break;
                    tc_fence_after();
                    issue_s(gg);
                }
                if (!ok) break;
                if (n <= NS) tc_commit(&q_empty[qb]);
                for (int j = 0; ok && j < n; ++j) {
                    const int gg = gk + j, st = gg % S, b = gg % NS;
                    if (!(ok = mbar_wait(&v_full[st], (gg / S) & 1, wc, 102))) break;
                    if (j == 0 && nq > 0 && !(ok = mbar_wait(o_free, (nq - 1) & 1, wc, 103))) break;
                    if (!(ok = mbar_wait(&p_full[b], (gg / NS) & 1, wc, 104))) break;
                    tc_fence_after();
                    const uint32_t v_addr = smem_u32(sV + st * C::kTileBytes);
                    const uint32_t p_addr = smem_u32(sP + b * C::kPBytes);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + C::kColO, sdesc_sw128(v_addr + kk * 2048, C::kKVSlab, 1024),
                               sdesc_sw128(p_addr + (kk >> 2) * C::kPSlab + (kk & 3) * 32, 16, 1024), id_pv,
                               (j > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&pv_done[b]);
                    tc_commit(&v_empty[st]);
                    // S^T of tile gg + NS into the columns of tile gg; P of that tile goes to
                    // the P buffer just read. The tensor core runs one thread's products in
                    // issue order.
                    if (j + NS < n) {
                        const int g2 = gg + NS;
                        if (!(ok = mbar_wait(&k_full[g2 % S], (g2 / S) & 1, wc, 105))) break;
                        tc_fence_after();
                        issue_s(g2);
                        if (j + NS + 1 == n) tc_commit(&q_empty[qb]);
                    }
                }
                tc_commit(o_ready);
                gk += n;
                ++nq;
            }
            tc_commit(mma_done);
            mbar_wait_drain(mma_done, 0);
            const uint32_t a = smem_u32(sm_done);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < 4000000000ull) {
            }
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax / epilogue
        // Thread l: key l of every tile (TMEM lane l of S^T) and d index l of O^T. The
        // four warps meet on mbarriers with one arrival per warp (bounded waits, so a
        // warp that gave up on a wait cannot leave the others stuck).
        const int w4 = warp - 4;
        const int l_idx = w4 * 32 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(w4 * 32) << 16);
        const uint32_t o_addr = lane_base + C::kColO;
        volatile int* flags = reinterpret_cast<volatile int*>(smem + C::kFlagOff);
        volatile float* red = reinterpret_cast<volatile float*>(smem + C::kRedOff);
        volatile float* sums = reinterpret_cast<volatile float*>(smem + C::kSumOff);
        uint64_t* xb_flag = sm_done + 1;     // [2] per tile parity
        uint64_t* xb_red = xb_flag + 2;      // [2] per tile parity, slow tiles only
        uint64_t* xb_sum = xb_red + 2;       // one per segment
        const float sl2 = args.scale_log2;
        const int g = args.group, R = args.R;
        // Meet the other three warps: this warp's shared-memory writes are visible to
        // them once every warp's wait returns.
        auto meet = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
            return warp_all(mbar_wait(bar, parity, wc, site));
        };
        int gk = 0, nq = 0;
        int n_red0 = 0, n_red1 = 0;  // uses of xb_red[0], xb_red[1] so far
        bool ok = true;
        for (DecItem it = rg.first; ok && it.P < rg.s_hi; it = dec_next<SEQLENS>(args, it, rg.T)) {
            int j0, n;
            if (!dec_segment(rg.s_lo, rg.s_hi, it, j0, n)) continue;
            // Row r (token r / g) sees keys below min(len, r / g + len - Nq + 1) under the
            // causal mask, below len otherwise.
            const int causal_base = it.len - args.Nq + 1;
            float m[RN], l[RN], lr[RN];
#pragma unroll
            for (int r = 0; r < RN; ++r) {
                m[r] = -INFINITY;
                l[r] = 0.f;
                lr[r] = 0.f;
            }
            for (int j = 0; j < n; ++j) {
                const int gg = gk + j, par = gg & 1, b = gg % NS;
                ok = warp_all(mbar_wait(&s_full[b], (gg / NS) & 1, wc, 106));
                if (!ok) break;
                tc_fence_after();
                uint32_t sv[32];
                tmem_ld32(lane_base + 32 * b, sv);
                tmem_ld_wait(sv);
                const int key = (j0 + j) * 128 + l_idx;
                float x[RN];
                bool exceed = false;
                int t = 0, hc = 0;
#pragma unroll
                for (int r = 0; r < RN; ++r) {
                    if (args.pair && r == args.r8) {  // the second KV head's rows start again at token 0
                        t = 0;
                        hc = 0;
                    }
                    const int khi = causal ? min(it.len, t + causal_base) : it.len;
                    x[r] = key < khi ? __uint_as_float(sv[r]) * sl2 : -INFINITY;
                    exceed |= x[r] > m[r] + kRescaleThreshold;
                    if (++hc == g) {
                        hc = 0;
                        ++t;
                    }
                }
                // Does any row need a new reference max? (Always on a row's first keys.)
                const bool wexc = __any_sync(0xffffffffu, exceed);
                if (lane == 0) flags[par * 4 + w4] = wexc ? 1 : 0;
                ok = meet(&xb_flag[par], (gg >> 1) & 1, 107);
                if (!ok) break;
                if (flags[par * 4] | flags[par * 4 + 1] | flags[par * 4 + 2] | flags[par * 4 + 3]) {
                    // The exact tile max of every row, then the reference moves there.
                    volatile float* rd = red + par * 4 * RN;
#pragma unroll
                    for (int r = 0; r < RN; ++r) {
                        float v = x[r];
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
                        if (lane == r) rd[w4 * RN + r] = v;
                    }
                    ok = meet(&xb_red[par], (par ? n_red1 : n_red0) & 1, 108);
                    if (par) ++n_red1; else ++n_red0;
                    if (!ok) break;
                    // O^T holds the products up to the previous tile once its P V is
                    // complete; it is rescaled with the normalisers (by 1 where a row's
                    // reference stays).
                    const bool with_o = j > 0;
                    uint32_t ov[32];
                    if (with_o) {  // P V of tile gg - 1: its buffer's use (gg - 1) / NS
                        ok = warp_all(mbar_wait(&pv_done[(gg - 1) % NS], ((gg - 1) / NS) & 1, wc, 109));
                        if (!ok) break;
                        tc_fence_after();
                        tmem_ld32(o_addr, ov);
                        tmem_ld_wait(ov);
                    }
#pragma unroll
                    for (int r = 0; r < RN; ++r) {
                        const float mx = fmaxf(fmaxf(rd[r], rd[RN + r]), fmaxf(rd[2 * RN + r], rd[3 * RN + r]));
                        float alpha = 1.f;
                        if (mx > m[r]) {
                            if (m[r] != -INFINITY) alpha = ex2_approx(m[r] - mx);
                            m[r] = mx;
                        }
                        l[r] *= alpha;
                        lr[r] *= alpha;
                        if (with_o) ov[r] = __float_as_uint(__uint_as_float(ov[r]) * alpha);
                    }
                    if (with_o) {
                        tmem_st32(o_addr, ov);
                        tmem_st_wait();
                    }
                }
                // P = 2^(x - m) rounded to 16 bits: row r, key l of P buffer b (free: S^T of
                // this tile complete implies P V of tile gg - NS complete).
                uint8_t* pb = sP + b * C::kPBytes;
#pragma unroll
                for (int r = 0; r < RN; r += 2) {
                    const float p0 = ex2_approx(x[r] + (m[r] == -INFINITY ? 0.f : -m[r]));
                    const float p1 = ex2_approx(x[r + 1] + (m[r + 1] == -INFINITY ? 0.f : -m[r + 1]));
                    l[r] += p0;
                    l[r + 1] += p1;
                    const uint32_t u = pack2<BF16>(p0, p1);
                    lr[r] += unpack_lo<BF16>(u);
                    lr[r + 1] += unpack_hi<BF16>(u);
                    *reinterpret_cast<uint16_t*>(pb + dec_p_offset<RN>(r, l_idx)) = static_cast<uint16_t>(u & 0xffffu);
                    *reinterpret_cast<uint16_t*>(pb + dec_p_offset<RN>(r + 1, l_idx)) = static_cast<uint16_t>(u >> 16);
                }
                // The sequence's last tile: rows of V past its end may hold anything
                // (0 x NaN would reach O); they are zeroed before P V reads them. V's
                // previous use of this buffer (tile gg - S, S >= NS) is complete: S^T of
                // this tile is, so P V of tile gg - NS is.
                if (SEQLENS && j0 + j == it.ntk - 1 && (it.len & 127) != 0) {
                    ok = warp_all(mbar_wait(&v_full[gg % S], (gg / S) & 1, wc, 110));
                    if (!ok) break;
                    const int v0 = it.len & 127;
                    const int per_slab = (128 - v0) * 8;
                    uint8_t* vt = sV + (gg % S) * C::kTileBytes;
                    for (int xx = l_idx; xx < per_slab * C::kSlabs; xx += 128) {
                        const int s = xx / per_slab, rem = xx % per_slab;
                        *reinterpret_cast<uint4*>(vt + s * C::kKVSlab + (v0 + rem / 8) * 128 + (rem % 8) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&p_full[b]);
            }
            if (!ok) break;
            // Row sums over the 128 keys' threads.
#pragma unroll
            for (int r = 0; r < RN; ++r) {
                float a = l[r], b = lr[r];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    a += __shfl_xor_sync(0xffffffffu, a, off);
                    b += __shfl_xor_sync(0xffffffffu, b, off);
                }
                if (lane == r) {
                    sums[(w4 * RN + r) * 2] = a;
                    sums[(w4 * RN + r) * 2 + 1] = b;
                }
            }
            ok = meet(xb_sum, nq & 1, 111);
            if (!ok) break;
            ok = warp_all(mbar_wait(o_ready, nq & 1, wc, 112));
            if (!ok) break;
            tc_fence_after();
            uint32_t ov[32];
            tmem_ld32(o_addr, ov);
            tmem_ld_wait(ov);
            const size_t slot = static_cast<size_t>(cta) + static_cast<size_t>(it.b) * args.Hkv + it.hk;
            // Partial row rp of tile row r; with paired KV heads the rows of head group k
            // sit in O^T lanes 64 k .. 64 k + 63 and partials have d = 64.
            const bool pair = args.pair != 0;
#pragma unroll
            for (int r = 0; r < RN; ++r) {
                const int k = (pair && r >= args.r8) ? 1 : 0;
                const int rl = r - k * args.r8;
                const bool valid = pair ? rl < args.rg : r < R;
                const int rp = pair ? k * args.rg + rl : r;
                if (valid) {
                    float lt = 0.f, lrt = 0.f;
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        lt += sums[(w * RN + r) * 2];
                        lrt += sums[(w * RN + r) * 2 + 1];
                    }
                    const float o_val = __uint_as_float(ov[r]) * (lrt > 0.f ? 1.f / lrt : 0.f);
                    if (pair) {
                        if ((l_idx >> 6) == k) args.o_part[(slot * R + rp) * 64 + (l_idx & 63)] = o_val;
                    } else if (l_idx < D) {
                        args.o_part[(slot * R + rp) * D + l_idx] = o_val;
                    }
                    if (l_idx == r) {
                        float L = -INFINITY;
                        if (lt > 0.f) {
                            float lg;
                            asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(lt));
                            L = (m[r] + lg) * kLn2;
                        }
                        args.lse_part[slot * R + rp] = L;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(o_free);
            gk += n;
            ++nq;
        }
        tc_fence_before();
        mbar_arrive(sm_done);
    }
}

// Merge of the segments of each item: one block of four warps per (item, row r) of
// the R rows: L = log sum_s exp(L_s) and O = sum_s exp(L_s - L) O_s over the CTAs
// whose tile range meets the item (warp w takes every fourth segment, lanes d in
// chunks of four), written to o [B, Nq, Hq, d] and lse [B, Hq, Nq]. An item without
// keys, or a row that sees none, gets O = 0 and L = -inf.
template <int D, bool BF16, bool SEQLENS>
__global__ void __launch_bounds__(128) fa_decode_combine(const DecodeArgs a) {
    // Launched as a programmatic dependent of the split kernel: everything below
    // reads what that kernel wrote, so wait for it to complete (no-op otherwise).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ float4 part[4][D / 4];
    const int lane = lane_id(), warp = warp_id();
    const int item = static_cast<int>(blockIdx.x / a.R), r = static_cast<int>(blockIdx.x % a.R);
    const int b = item / a.Hkv, hk = item % a.Hkv;
    const int len = dec_len<SEQLENS>(a, b);
    const int ntk = (len + 127) / 128;
    long long T = 0, P = 0;
    if (ntk > 0) {
        if constexpr (SEQLENS) {  // written by the split kernel, which runs whenever some item has keys
            T = a.meta[0];
            P = a.meta[1 + item];
        } else {
            T = static_cast<long long>(a.B) * a.Hkv * (ntk + kDecItemCost);
            P = static_cast<long long>(item) * (ntk + kDecItemCost);
        }
    }
    // The CTAs whose cost range holds one of the item's tiles (units P + kDecItemCost ..).
    int c0 = 0, c1 = -1;
    if (ntk > 0 && T > 0) {
        c0 = dec_cta_of(P + kDecItemCost, T, a.G);
        c1 = dec_cta_of(P + kDecItemCost + ntk - 1, T, a.G);
    }
    // CTA c's range is empty only when there are fewer tiles than CTAs.
    const bool all_have = T >= a.G;
    auto has = [&](int c) { return all_have || dec_split(c, T, a.G) < dec_split(c + 1, T, a.G); };
    const float* lp = a.lse_part + static_cast<size_t>(item) * a.R + r;  // segment of CTA c: lp[c * R]
    // Every warp finds the max and the sum of weights itself (lanes over segments).
    float Lm = -INFINITY;
    for (int c = c0 + lane; c <= c1; c += 32)
        if (has(c)) Lm = fmaxf(Lm, lp[static_cast<size_t>(c) * a.R]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) Lm = fmaxf(Lm, __shfl_xor_sync(0xffffffffu, Lm, off));
    float wsum = 0.f;
    if (Lm != -INFINITY)
        for (int c = c0 + lane; c <= c1; c += 32)
            if (has(c)) wsum += expf(lp[static_cast<size_t>(c) * a.R] - Lm);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (Lm != -INFINITY && lane < D / 4) {
#pragma unroll 2
        for (int c = c0 + warp; c <= c1; c += 4) {
            if (!has(c)) continue;
            const size_t row = (static_cast<size_t>(c) + item) * a.R + r;
            const float w = expf(a.lse_part[row] - Lm);
            const float4 x = reinterpret_cast<const float4*>(a.o_part + row * D)[lane];
            acc.x += w * x.x;
            acc.y += w * x.y;
            acc.z += w * x.z;
            acc.w += w * x.w;
        }
    }
    if (lane < D / 4) part[warp][lane] = acc;
    __syncthreads();
    if (warp != 0 || lane >= D / 4) return;
#pragma unroll
    for (int w = 1; w < 4; ++w) {
        const float4 y = part[w][lane];
        acc.x += y.x;
        acc.y += y.y;
        acc.z += y.z;
        acc.w += y.w;
    }
    // Row r of the item: with paired KV heads rows 0..rg-1 belong to KV head 2 hk and
    // rows rg..2 rg-1 to KV head 2 hk + 1.
    const int kv = a.pair ? 2 * hk + r / a.rg : hk;
    const int rl = a.pair ? r % a.rg : r;
    const int t = rl / a.group, h = kv * a.group + rl % a.group;
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint16_t* o = static_cast<uint16_t*>(a.o) + ((static_cast<size_t>(b) * a.Nq + t) * a.Hq + h) * D + lane * 4;
    *reinterpret_cast<uint2*>(o) = make_uint2(pack2<BF16>(acc.x * inv, acc.y * inv), pack2<BF16>(acc.z * inv, acc.w * inv));
    if (lane == 0)
        a.lse[(static_cast<size_t>(b) * a.Hq + h) * a.Nq + t] = wsum > 0.f ? Lm + logf(wsum) : -INFINITY;
}

}  // namespace fa
