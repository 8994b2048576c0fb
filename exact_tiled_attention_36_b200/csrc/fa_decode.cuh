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

// One item (sequence b, KV head hk): its keys and its first tile in the sequence of T.
struct DecItem {
    int b, hk, len, ntk;
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
    return it;
}

// The item after `it`; past the last one P = T (the walk ends there).
template <bool SEQLENS>
__device__ __forceinline__ DecItem dec_next(const DecodeArgs& a, const DecItem& it, long long T) {
    if (it.hk + 1 < a.Hkv) return dec_item<SEQLENS>(a, it.b, it.hk + 1, it.P + it.ntk);
    if (it.b + 1 < a.B) return dec_item<SEQLENS>(a, it.b + 1, 0, it.P + it.ntk);
    DecItem e = it;
    e.P = T;
    e.ntk = 0;
    return e;
}

// CTA whose tile range holds tile t: the largest c with floor(c T / G) <= t.
__device__ __forceinline__ int dec_cta_of(long long t, long long T, int G) {
    return static_cast<int>(((t + 1) * G - 1) / T);
}

__device__ __forceinline__ long long dec_split(int c, long long T, int G) { return (static_cast<long long>(c) * T) / G; }

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
    const int G = args.G;
    const int cta = static_cast<int>(blockIdx.x);
    const int tid = static_cast<int>(threadIdx.x);
    const int warp = warp_id();
    const int lane = lane_id();
    uint8_t* misc = smem + C::kMiscOff;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(misc);
    int* abort_flag = reinterpret_cast<int*>(misc + 4);

    // ---------------------------------------------------------------- the CTA's tiles
    // T and the item holding the CTA's first tile. With sequence lengths every CTA
    // sums the per-sequence tile counts itself (a block reduction, then a block scan
    // that stops at the sequence holding that tile).
    long long T, s_lo, s_hi;
    int b0;
    long long P0;  // first tile of sequence b0 (its KV head 0)
    if constexpr (SEQLENS) {
        int* found = reinterpret_cast<int*>(misc + 8);
        long long* sh_T = reinterpret_cast<long long*>(misc + 16);
        int* sh_b0 = reinterpret_cast<int*>(misc + 24);
        long long* sh_P0 = reinterpret_cast<long long*>(misc + 32);
        long long* ws = reinterpret_cast<long long*>(misc + 48);  // [8] per-warp sums
        auto tiles_of = [&](int b) -> long long {
            return b < args.B ? static_cast<long long>(args.Hkv) * ((dec_len<true>(args, b) + 127) / 128) : 0;
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
        for (int w = 0; w < kDecThreads / 32; ++w) T += ws[w];
        if (cta == 0 && tid == 0) args.meta[0] = T;
        s_lo = dec_split(cta, T, G);
        s_hi = dec_split(cta + 1, T, G);
        if (s_lo >= s_hi) return;  // no tile for this CTA (fewer tiles than CTAs)
        __syncthreads();           // every thread has read ws
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
            for (int w = 0; w < kDecThreads / 32; ++w) {
                const long long y = ws[w];
                if (w < warp) before += y;
                total += y;
            }
            const long long excl = run + before + incl - x;
            if (x > 0 && excl <= s_lo && s_lo < excl + x) {
                *sh_b0 = b;
                *sh_P0 = excl;
                *found = 1;
            }
            __syncthreads();
            if (*found) break;
            run += total;
        }
        if (!*found) return;  // cannot happen: s_lo < T
        b0 = *sh_b0;
        P0 = *sh_P0;
        (void)sh_T;
    } else {
        const long long per_b = static_cast<long long>(args.Hkv) * ((args.Nk + 127) / 128);
        T = per_b * args.B;
        s_lo = dec_split(cta, T, G);
        s_hi = dec_split(cta + 1, T, G);
        if (s_lo >= s_hi) return;
        b0 = static_cast<int>(s_lo / per_b);
        P0 = b0 * per_b;
    }
    // The item holding tile s_lo; every role walks the items from here.
    const DecItem first = [&] {
        const int ntk = (dec_len<SEQLENS>(args, b0) + 127) / 128;
        const int hk = static_cast<int>((s_lo - P0) / ntk);
        return dec_item<SEQLENS>(args, b0, hk, P0 + static_cast<long long>(hk) * ntk);
    }();

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
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            constexpr uint32_t kQBytesPerRow = C::kSlabs * 128;
            int gk = 0, nq = 0, k_issued = 0, v_issued = 0;
            bool ok = true;
            // One K or V tile (key tile kt of item `it`) into ring buffer `dst`.
            auto load_kv = [&](uint8_t* dst, const CUtensorMap* m, uint64_t* bar, const DecItem& it, int kt) {
                if constexpr (!PAGED) {
                    mbar_arrive_expect_tx(bar, C::kTileBytes);
#pragma unroll
                    for (int s = 0; s < C::kSlabs; ++s)
                        tma_load_4d(dst + s * C::kSlabBytes, m, bar, s * 64, it.hk, kt * 128, it.b);
                } else {
                    // Boxes of page_box rows (one page holds whole boxes); boxes past the
                    // sequence's end are not loaded (their rows are masked and zeroed).
                    const int pb = args.page_box;
                    const int keys = min(128, it.len - kt * 128);
                    const int boxes = (keys + pb - 1) / pb;
                    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(boxes * pb * 128 * C::kSlabs));
                    const int* bt = args.block_table + static_cast<size_t>(it.b) * args.max_pages;
                    for (int x = 0; x < boxes; ++x) {
                        const int key = kt * 128 + x * pb;
                        const int page = bt[key / args.page_size];
#pragma unroll
                        for (int s = 0; s < C::kSlabs; ++s)
                            tma_load_4d(dst + s * C::kSlabBytes + x * pb * 128, m, bar, s * 64, it.hk,
                                        key % args.page_size, page);
                    }
                }
            };
            for (DecItem it = first; ok && it.P < s_hi; it = dec_next<SEQLENS>(args, it, T)) {
                const long long lo = max(s_lo, it.P), hi = min(s_hi, it.P + it.ntk);
                if (lo >= hi) continue;
                const int j0 = static_cast<int>(lo - it.P), n = static_cast<int>(hi - lo);
                if (SEQLENS && lo == it.P) args.meta[1 + static_cast<size_t>(it.b) * args.Hkv + it.hk] = it.P;
                // Q of the group once the previous segment's last S product has read Q.
                if (!(ok = mbar_wait(q_empty, (nq & 1) ^ 1u, wc, 80))) break;
                mbar_arrive_expect_tx(q_full, kQBytesPerRow * args.R);
                for (int k = 0; k < args.nb; ++k)
#pragma unroll
                    for (int s = 0; s < C::kSlabs; ++s)
                        tma_load_4d(sQ + s * C::kSlabBytes + (args.nb > 1 ? k * 4096 : 0), &tm_q, q_full, s * 64,
                                    it.hk * g + k * args.gh, 0, it.b);
                ++nq;
                for (int j = 0; j < n; ++j) {
                    const int gg = gk + j, st = gg % S;
                    const uint32_t ph = (gg / S) & 1;
                    if (!(ok = mbar_wait(&k_empty[st], ph ^ 1u, wc, 81))) break;
                    load_kv(sK + st * C::kTileBytes, &tm_k, &k_full[st], it, j0 + j);
                    ++k_issued;
                    if (!(ok = mbar_wait(&v_empty[st], ph ^ 1u, wc, 82))) break;
                    load_kv(sV + st * C::kTileBytes, &tm_v, &v_full[st], it, j0 + j);
                    ++v_issued;
                }
                gk += n;
            }
            if (nq > 0) mbar_wait_drain(q_full, (nq - 1) & 1);
            for (int st = 0; st < S; ++st) {
                if (k_issued > st) mbar_wait_drain(&k_full[st], ((st + S * ((k_issued - 1 - st) / S)) / S) & 1);
                if (v_issued > st) mbar_wait_drain(&v_full[st], ((st + S * ((v_issued - 1 - st) / S)) / S) & 1);
            }
        }
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
                const long long lo = max(s_lo, it.P), hi = min(s_hi, it.P + it.ntk);
                if (lo >= hi) continue;
                const int n = static_cast<int>(hi - lo);
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
            const long long lo = max(s_lo, it.P), hi = min(s_hi, it.P + it.ntk);
            if (lo >= hi) continue;
            const int j0 = static_cast<int>(lo - it.P), n = static_cast<int>(hi - lo);
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

// Merge of the segments of one item per CTA: for each of its R rows,
// L = log sum_s exp(L_s) and O = sum_s exp(L_s - L) O_s over the CTAs whose tile
// range meets the item, written to o [B, Nq, Hq, d] and lse [B, Hq, Nq]. An item
// without keys, or a row that sees none, gets O = 0 and L = -inf.
template <int D, bool BF16, bool SEQLENS>
__global__ void __launch_bounds__(128) fa_decode_combine(const DecodeArgs a) {
    const int item = static_cast<int>(blockIdx.x);
    const int b = item / a.Hkv, hk = item % a.Hkv;
    const int len = dec_len<SEQLENS>(a, b);
    const int ntk = (len + 127) / 128;
    long long T, P;
    if constexpr (SEQLENS) {  // written by the split kernel (which runs whenever some item has keys)
        T = ntk > 0 ? a.meta[0] : 0;
        P = ntk > 0 ? a.meta[1 + item] : 0;
    } else {
        T = static_cast<long long>(a.B) * a.Hkv * ntk;
        P = static_cast<long long>(item) * ntk;
    }
    int c0 = 0, c1 = -1;
    if (ntk > 0 && T > 0) {
        c0 = dec_cta_of(P, T, a.G);
        c1 = dec_cta_of(P + ntk - 1, T, a.G);
    }
    uint16_t* o = static_cast<uint16_t*>(a.o);
    for (int idx = static_cast<int>(threadIdx.x); idx < a.R * (D / 8); idx += static_cast<int>(blockDim.x)) {
        const int r = idx / (D / 8), c8 = idx % (D / 8);
        const int t = r / a.group, h = hk * a.group + r % a.group;
        float Lm = -INFINITY;
        for (int c = c0; c <= c1; ++c)
            if (dec_split(c, T, a.G) < dec_split(c + 1, T, a.G))
                Lm = fmaxf(Lm, a.lse_part[static_cast<size_t>(c + item) * a.R + r]);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float wsum = 0.f;
        if (Lm != -INFINITY) {
            for (int c = c0; c <= c1; ++c) {
                if (dec_split(c, T, a.G) >= dec_split(c + 1, T, a.G)) continue;
                const size_t row = static_cast<size_t>(c + item) * a.R + r;
                const float w = expf(a.lse_part[row] - Lm);
                if (w == 0.f) continue;
                wsum += w;
                const float4* src = reinterpret_cast<const float4*>(a.o_part + row * D + c8 * 8);
                const float4 x0 = src[0], x1 = src[1];
                acc[0] += w * x0.x;
                acc[1] += w * x0.y;
                acc[2] += w * x0.z;
                acc[3] += w * x0.w;
                acc[4] += w * x1.x;
                acc[5] += w * x1.y;
                acc[6] += w * x1.z;
                acc[7] += w * x1.w;
            }
        }
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
        uint32_t pk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) pk[i] = pack2<BF16>(acc[2 * i] * inv, acc[2 * i + 1] * inv);
        const size_t orow = (static_cast<size_t>(b) * a.Nq + t) * a.Hq + h;
        *reinterpret_cast<uint4*>(o + orow * D + c8 * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        if (c8 == 0)
            a.lse[(static_cast<size_t>(b) * a.Hq + h) * a.Nq + t] = wsum > 0.f ? Lm + logf(wsum) : -INFINITY;
    }
}

}  // namespace fa
