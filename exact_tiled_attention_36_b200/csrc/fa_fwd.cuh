// fa_fwd.cuh: tiled exact attention forward for sm_100a, persistent CTAs with
// two query tiles per work unit.
//
// A work unit is two 128-row query tiles Q_0, Q_1 (rows q0 .. q0 + 255) of one
// (batch, query head); the unit walks the key/value tiles K_j, V_j of 128 rows
// with the online softmax ("FlashAttention/zh", section "FlashAttention
// algorithm": S_ij = Q_i K_j^T, running row max m and normaliser l, rescale of
// the partial output by exp(m_old - m_new), final O_i / l_i and L_i = m_i +
// log l_i), query tiles outside and key tiles inside (the FlashAttention-2
// split, section "variants"). Every K/V tile loaded serves both query tiles,
// and the softmax of one tile overlaps the tensor-core work of the other.
//
// Persistent tile scheduler: the grid has at most one CTA per SM and CTA c
// takes units c, 2G - 1 - c, 2G + c, ... of a fixed unit order (G CTAs; the
// order alternates direction every round). Without the causal mask the order
// keeps the units of one (batch, head) together so neighbouring CTAs share K/V
// in the L2; under the causal mask it runs the heaviest units (the last query
// rows) first. The CTA keeps its barriers, TMEM and K/V ring from unit to
// unit: the producer loads the next unit's Q as soon as the current unit's
// last S product has been issued, and the MMA threads issue the next unit's
// first S products while the softmax warpgroups write the current unit's O.
//
// Warp roles (384 threads):
//   warp 0        TMA producer: Q_0, Q_1 per unit, K_j, V_j into 2-stage (d = 128)
//                 or 4-stage (d = 64) mbarrier rings that run across units.
//   warp 1        TMEM allocation and (d = 128) the single MMA-issuing thread. Per
//                 key tile j it issues O_0 += P_0 V_j, S_0 = Q_0 K_{j+1}^T,
//                 O_1 += P_1 V_j, S_1 = Q_1 K_{j+1}^T. S_t reuses the columns P_t
//                 was read from with no wait in between: the tensor core executes
//                 one thread's tcgen05.mma operations in issue order (the order
//                 NVIDIA's own Blackwell attention example relies on; the GPU
//                 parity tests check it).
//   warps 1, 2    (d = 64) one MMA-issuing thread per query tile, each on its own SM
//                 sub-partition: thread t issues S_t of key tile j + 1 as soon as
//                 the softmax has read S_t(j) (P_t has its own TMEM columns), then
//                 P_t V_j. Q and the K / V ring slots serve both tiles: their
//                 release barriers count one commit from each thread.
//   warps 4-7     softmax of tile 0; warps 8-11 softmax of tile 1. Thread r owns
//                 query row r of its tile (TMEM lane r) and keeps the whole row of
//                 S in registers: warps 0-3 hand registers over with setmaxnreg
//                 (80 each) so that the softmax threads get 208. P =
//                 2^(S scale log2 e - m) is formed with the scale folded into one
//                 FFMA and written as 16-bit pairs over the first half of S's
//                 columns. l (exact fp32) gives L; the sum of the rounded P
//                 normalises O, so the weights applied to V sum to one. O is
//                 rescaled in TMEM only when m has grown by more than 2^8 since
//                 the last rescale (exact: O and l share the reference max).
//                 After the unit's last product each warpgroup writes its O_t
//                 and L and releases O_t's columns for the next unit.
//   warps 2-3     idle (d = 128); warp 3 idle (d = 64).
//
// TMEM columns: [0,128) S_0 / P_0, [128,256) S_1 / P_1, [256,256+d) O_0,
// [256+d,256+2d) O_1. With d = 64, P_t has its own columns [384 + 64 t, 448 + 64 t)
// instead: the softmax frees S_t as soon as it has read it (s_free), the MMA thread
// issues S_t of the next key tile into it at once, and the P_t V product signals
// pv_done, which the softmax waits for before it writes the next P_t or rescales O_t.
// The softmax of consecutive key tiles then no longer waits for the P V and S
// products in between (at d = 64 its exponentials outweigh the products).
#pragma once

#include "sm100.cuh"

namespace fa {

struct FwdArgs {
    void* o;
    float* lse;
    const int* cu_q;  // varlen: [num_batches + 1]
    const int* cu_k;
    int num_batches;  // B, or the number of sequences
    int total_q;      // varlen: rows of the q/o buffers (no row at or past it is written)
    int Hq;
    int group;        // Hq / Hkv
    int Nq;           // fixed: sequence lengths; varlen: max_seqlen bounds
    int Nk;
    long long o_sb, o_ss, o_sh;  // O strides in elements: batch, token, head (d is contiguous)
    int wl, wr;       // MASKED: keys from wl before to wr after the aligned diagonal (< 0: unbounded)
    int n_anchor;     // kMaskAnchor: keys 0 .. n_anchor - 1 are visible below the window too
    // Key mask (null: none): bit j % 32 of word b * kb_words + j / 32 set = key j of batch b
    // is visible (ANDed with the mask kind).
    const uint32_t* key_bits;
    int kb_words;
    int nu;           // units (256 query rows) per sequence: ceil(Nq / 256)
    int n_units;      // nu * Hq * num_batches
    float scale_log2;  // scale * log2(e)
    float norm_eps;    // QK RMS normalisation (fa_fwd_qk_rmsnorm): epsilon
    // FP8 (E4M3 Q, K, V): dequantisation factors per 128-token block of one head,
    // q_scale [B, Hq, nqb], k_scale and v_scale [B, Hkv, nkb].
    const float* q_scale;
    const float* k_scale;
    const float* v_scale;
    int nqb, nkb;
    int* err;
};


// FP8: one-byte elements (a 128-row tile of d = 128 is a single 128-byte-wide slab).
template <int D, bool FP8 = false>
struct FwdCfg {
    static constexpr int kElemBytes = FP8 ? 1 : 2;
    static constexpr int kSlabElems = 128 / kElemBytes;  // columns per 128-byte slab
    static constexpr int kSlabs = D * kElemBytes / 128;
    static constexpr int kSlabBytes = 128 * 128;
    static constexpr int kTileBytes = kSlabs * kSlabBytes;  // 128 rows x d
    static constexpr int kKSteps = D * kElemBytes / 32;    // 32 bytes of K per MMA instruction
    static constexpr int kStages = FP8 ? 4 : ((D == 128) ? 2 : 4);
    static constexpr int kQOff = 0;                          // Q_0, Q_1
    static constexpr int kKOff = kQOff + 2 * kTileBytes;
    static constexpr int kVOff = kKOff + kStages * kTileBytes;
    // Epilogue staging: 2 KB per softmax warp (32 rows x 32 columns of O in 16 bits).
    static constexpr int kEpiOff = kVOff + kStages * kTileBytes;
    static constexpr int kEpiBytesPerWarp = 32 * 32 * 2;
    static constexpr int kBarOff = kEpiOff + 8 * kEpiBytesPerWarp;
    static constexpr int kNumBars = 2 + 4 * kStages + 2 + 2 + 2 + 2 + 1 + 1 + 1 + 2 + 2;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0, kColO = 256;  // S_t at 128 t, O_t at 256 + d t
    // d = 64 (16-bit): P_t has columns of its own, [384 + 64 t, 448 + 64 t), so S_t of
    // the next key tile can be computed while the softmax still works on this one.
    static constexpr bool kSepP = D == 64 && !FP8;
    static constexpr uint32_t kColP = kSepP ? 384 : 0;
    static_assert(!kSepP || kColP + 128 <= kTmemCols, "TMEM budget");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

constexpr int kFwdThreads = 384;
constexpr int kFwdRegsOther = 80;     // warps 0-3 after the split
constexpr int kFwdRegsSoftmax = 208;  // warps 4-11 after the split
// Registers at launch needed for the split to fit the CTA's pool.
constexpr int kFwdMinLaunchRegs = (128 * kFwdRegsOther + 256 * kFwdRegsSoftmax + kFwdThreads - 1) / kFwdThreads;

// Everything one role needs to know about a work unit; every role decodes the
// same units in the same order.
struct FwdUnit {
    int h, bidx, q0;
    int q_len, k_len, q_row0, k_row0, tma_b;
    int jlo, n_kv;       // the unit walks key tiles jlo .. jlo + n_kv - 1 (steps 0 .. n_kv - 1)
    int a0, b0, a1, b1;  // query tile t is active on steps a_t .. b_t - 1 (none if a_t == b_t)
    bool rows;           // the unit holds at least one query row
    // kMaskAnchor: the walk is the anchor tiles 0 .. na - 1, then window tiles from jw
    // (step s >= na is tile jw + s - na); query tile t sees anchor tiles 0 .. ta_t - 1
    // and its window's tiles [jl_t, jh_t).
    int na, jw, ta0, ta1, jl0, jh0, jl1, jh1;
    __device__ __forceinline__ int a(int t) const { return t ? a1 : a0; }
    __device__ __forceinline__ int b(int t) const { return t ? b1 : b0; }
    __device__ __forceinline__ int ta(int t) const { return t ? ta1 : ta0; }
    __device__ __forceinline__ int jl(int t) const { return t ? jl1 : jl0; }
    __device__ __forceinline__ int jh(int t) const { return t ? jh1 : jh0; }
};

// 16-byte shared-memory accesses by 32-bit shared address.
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr) : "memory");
    return v;
}

// Mask kinds of the forward: none, causal (the window (-1, 0), fixed at compile
// time), the sliding window (wl, wr) of FwdArgs, or that window plus the global
// anchor keys 0 .. n_anchor - 1 (visible to a query whenever the window's right
// bound allows them).
enum : int { kMaskNone = 0, kMaskCausal = 1, kMaskWindow = 2, kMaskAnchor = 3 };

// First visible key and one past the last for query q (bottom-right alignment).
template <int MASK>
__device__ __forceinline__ void key_range(const FwdArgs& a, int q, int q_len, int k_len, int& lo, int& hi) {
    lo = 0;
    hi = k_len;
    const int aligned = q + k_len - q_len;
    if (MASK == kMaskCausal) hi = min(k_len, aligned + 1);
    if (MASK == kMaskWindow || MASK == kMaskAnchor) {
        if (a.wl >= 0) lo = max(0, aligned - a.wl);
        if (a.wr >= 0) hi = min(k_len, aligned + a.wr + 1);
    }
}

template <int MASK, bool VARLEN>
__device__ __forceinline__ FwdUnit fwd_unit(int u, const FwdArgs& a) {
    FwdUnit w;
    const int hb = a.Hq * a.num_batches;
    int unit, r;
    if (MASK == kMaskCausal) {  // heaviest units (last query rows) first
        unit = a.nu - 1 - u / hb;
        r = u % hb;
    } else {  // the units of one (batch, head) together
        unit = u % a.nu;
        r = u / a.nu;
    }
    w.h = r % a.Hq;
    w.bidx = r / a.Hq;
    w.q0 = unit * 256;
    if constexpr (VARLEN) {
        w.q_row0 = a.cu_q[w.bidx];
        w.k_row0 = a.cu_k[w.bidx];
        w.q_len = min(a.cu_q[w.bidx + 1] - w.q_row0, a.Nq);
        w.k_len = min(a.cu_k[w.bidx + 1] - w.k_row0, a.Nk);
        w.tma_b = 0;
    } else {
        w.q_row0 = 0;
        w.k_row0 = 0;
        w.q_len = a.Nq;
        w.k_len = a.Nk;
        w.tma_b = w.bidx;
    }
    w.rows = w.q0 < w.q_len;
    // Key tiles [jl[t], jh[t]) query tile t (rows q0 + 128 t ..) needs: the window of its
    // first row starts lowest, that of its last row ends highest.
    auto tiles = [&](int qt, int& jl, int& jh) {
        jl = jh = 0;
        if (qt >= w.q_len) return;
        int lo, hi, lo2, hi2;
        key_range<MASK>(a, qt, w.q_len, w.k_len, lo, hi);
        key_range<MASK>(a, min(qt + 127, w.q_len - 1), w.q_len, w.k_len, lo2, hi2);
        if (hi2 > lo) {
            jl = lo / 128;
            jh = (hi2 + 127) / 128;
        }
    };
    int jl0, jh0, jl1, jh1;
    tiles(w.q0, jl0, jh0);
    tiles(w.q0 + 128, jl1, jh1);
    if constexpr (MASK == kMaskAnchor) {
        // Anchor tiles of query tile t: keys below n_anchor and below the largest
        // right bound of its rows (its last row's).
        auto anchors = [&](int qt) -> int {
            if (qt >= w.q_len) return 0;
            int lo, hi;
            key_range<MASK>(a, min(qt + 127, w.q_len - 1), w.q_len, w.k_len, lo, hi);
            return (min(a.n_anchor, hi) + 127) / 128;
        };
        w.ta0 = anchors(w.q0);
        w.ta1 = anchors(w.q0 + 128);
        w.jl0 = jl0;
        w.jh0 = jh0;
        w.jl1 = jl1;
        w.jh1 = jh1;
        w.na = max(w.ta0, w.ta1);
        const bool f0 = jh0 == jl0, f1 = jh1 == jl1;
        const int wlo = f0 ? jl1 : (f1 ? jl0 : min(jl0, jl1));
        const int whi = f0 ? jh1 : (f1 ? jh0 : max(jh0, jh1));
        w.jw = max(w.na, wlo);
        w.jlo = 0;
        w.n_kv = w.na + max(0, whi - w.jw);
        w.a0 = w.b0 = w.a1 = w.b1 = 0;
        return w;
    }
    const bool e0 = jh0 == jl0, e1 = jh1 == jl1;
    w.jlo = e0 ? jl1 : (e1 ? jl0 : min(jl0, jl1));
    const int jhi = e0 ? jh1 : (e1 ? jh0 : max(jh0, jh1));
    w.n_kv = jhi - w.jlo;
    w.a0 = e0 ? 0 : jl0 - w.jlo;
    w.b0 = e0 ? 0 : jh0 - w.jlo;
    w.a1 = e1 ? 0 : jl1 - w.jlo;
    w.b1 = e1 ? 0 : jh1 - w.jlo;
    return w;
}

// Key tile of step s of the unit's walk.
template <int MASK>
__device__ __forceinline__ int fwd_tile(const FwdUnit& w, int s) {
    if constexpr (MASK == kMaskAnchor) return s < w.na ? s : w.jw + s - w.na;
    return w.jlo + s;
}

// Query tile t takes part in step s of the walk.
template <int MASK>
__device__ __forceinline__ bool fwd_active(const FwdUnit& w, int t, int s) {
    if constexpr (MASK == kMaskAnchor) {
        const int kt = fwd_tile<MASK>(w, s);
        return kt < w.ta(t) || (kt >= w.jl(t) && kt < w.jh(t));
    }
    return s >= w.a(t) && s < w.b(t);
}

// Number of steps query tile t takes part in, and the key tile of its j-th (anchor
// tiles first, then the window's tiles past them).
template <int MASK>
__device__ __forceinline__ int fwd_tile_steps(const FwdUnit& w, int t) {
    if constexpr (MASK == kMaskAnchor) return w.ta(t) + max(0, w.jh(t) - max(w.jl(t), w.ta(t)));
    return w.b(t) - w.a(t);
}
template <int MASK>
__device__ __forceinline__ int fwd_tile_of(const FwdUnit& w, int t, int j) {
    if constexpr (MASK == kMaskAnchor) return j < w.ta(t) ? j : max(w.jl(t), w.ta(t)) + j - w.ta(t);
    return w.jlo + w.a(t) + j;
}

// Unit of round k for CTA c of G: the direction alternates every round.
__device__ __forceinline__ int fwd_unit_index(int k, int c, int G) { return k * G + ((k & 1) ? G - 1 - c : c); }

// RMS normalisation, in place, of row r of a 128-row tile in shared memory (the
// 128-byte-swizzled layout of the TMA loads: 64-column slabs of 128-byte rows,
// 16-byte chunk c of row r at chunk c ^ (r % 8)): x <- x / sqrt(mean(x^2) + eps),
// unit gain, fp32 arithmetic, rounded to the 16-bit type.
template <int D, bool BF16>
__device__ __forceinline__ void rms_normalise_row(uint8_t* tile, int r, float eps) {
    constexpr int kSlabs = D / 64;
    // Sum of squares: pairs of elements through the packed f32x2 FMA into four
    // independent accumulators, one 64-column slab (8 chunks) loaded at a time.
    uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int s = 0; s < kSlabs; ++s) {
        uint4 x[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
            x[c] = *reinterpret_cast<const uint4*>(tile + s * 16384 + r * 128 + ((c ^ (r & 7)) << 4));
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint32_t w[4] = {x[c].x, x[c].y, x[c].z, x[c].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint64_t p = f2_pack(unpack_lo<BF16>(w[i]), unpack_hi<BF16>(w[i]));
                acc[i] = f2_fma(p, p, acc[i]);
            }
        }
    }
    const float ss = f2_sum(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])));
    const float inv = rsqrtf(ss * (1.f / D) + eps);
    const uint64_t inv2 = f2_pack(inv, inv);
#pragma unroll
    for (int s = 0; s < kSlabs; ++s)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint4* ptr = reinterpret_cast<uint4*>(tile + s * 16384 + r * 128 + ((c ^ (r & 7)) << 4));
            const uint4 x = *ptr;
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float lo, hi;
                f2_unpack(f2_mul(f2_pack(unpack_lo<BF16>(w[i]), unpack_hi<BF16>(w[i])), inv2), lo, hi);
                o[i] = pack2<BF16>(lo, hi);
            }
            *ptr = make_uint4(o[0], o[1], o[2], o[3]);
        }
}

// MASK: kMaskNone, kMaskCausal (bottom-right, folded at compile time), kMaskWindow
// (the sliding window (wl, wr) of FwdArgs) or kMaskAnchor (that window plus the
// anchor keys 0 .. n_anchor - 1); under VARLEN all of them apply within each sequence.
// QKNORM: Q arrives raw and each softmax thread RMS-normalises its own row of Q in
// shared memory (over d) at the start of a unit, before the tensor core reads it;
// K arrives normalised (fa_fwd_qk_rmsnorm runs fa_rms_normalise_rows over K first:
// every CTA would otherwise redo each K tile once per unit).
// FP8: Q, K, V are E4M3 with per-block dequantisation factors (fixed length, d = 128):
// S and P V run as kind::f8f6f4 products; the Q and K block factors join the exp2
// factor of each (query tile, key tile) pair, and V's block factor v_j enters P as
// 2^(log2(v_j / v_max)) before P is rounded to E4M3 (P <= 2^8 under the lazy
// rescale, inside E4M3's range), so O = v_max * sum(P' V) / l. O is bf16.
// KEYMASK: args.key_bits masks keys too (a compile-time switch, so that the other
// instantiations carry none of its per-tile work).
template <int D, bool BF16, int MASK, bool VARLEN, bool QKNORM, bool FP8 = false, bool KEYMASK = false>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdArgs args) {
    static_assert(!FP8 || (D == 128 && BF16 && !VARLEN && !QKNORM && MASK <= kMaskCausal), "FP8 forward shape");
    using C = FwdCfg<D, FP8>;
    constexpr int S = C::kStages;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (!smem_base_ok(smem, args.err)) return;
    const int G = static_cast<int>(gridDim.x);
    const int cta = static_cast<int>(blockIdx.x);

    using T16 = uint16_t;
    T16* o_base = static_cast<T16*>(args.o);
    uint8_t* sQ = smem + C::kQOff;
    uint8_t* sK = smem + C::kKOff;
    uint8_t* sV = smem + C::kVOff;
    uint8_t* sEpi = smem + C::kEpiOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* q_full = bars;
    uint64_t* q_empty = bars + 1;  // the unit's last S product has read Q
    uint64_t* k_full = bars + 2;
    uint64_t* k_empty = k_full + S;
    uint64_t* v_full = k_empty + S;
    uint64_t* v_empty = v_full + S;
    uint64_t* s_full = v_empty + S;  // [2 tiles]
    uint64_t* p_full = s_full + 2;   // [2]
    uint64_t* o_free = p_full + 2;   // [2] the epilogue has read O_t
    uint64_t* o_ready = o_free + 2;  // [2] every product of the unit's tile t is complete
    uint64_t* sm_done = o_ready + 2;  // every softmax thread is past its last TMEM access
    uint64_t* mma_done = sm_done + 1;  // every product this CTA issued is complete (both issuers)
    uint64_t* q_norm = mma_done + 1;   // QKNORM: Q of the unit normalised
    uint64_t* s_free = q_norm + 1;     // [2] kSepP: the softmax has read S_t
    uint64_t* pv_done = s_free + 2;    // [2] kSepP: P_t V is complete
    // The barrier the MMA thread waits on before reading Q.
    uint64_t* q_ready = QKNORM ? q_norm : q_full;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    int* abort_flag = reinterpret_cast<int*>(smem + C::kMiscOff + 4);

    const int warp = warp_id();
    const int lane = lane_id();

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        // d = 64 has two MMA-issuing threads (one per query tile); each commits once
        constexpr uint32_t kIssuers = C::kSepP ? 2 : 1;
        mbar_init(q_empty, kIssuers);
        for (int i = 0; i < S; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], kIssuers);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], kIssuers);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 128);
            mbar_init(&o_free[i], 128);
        }
        for (int i = 0; i < 2; ++i) mbar_init(&o_ready[i], 1);
        mbar_init(sm_done, 256);
        mbar_init(mma_done, kIssuers);
        mbar_init(q_norm, 256);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_free[i], 128);
            mbar_init(&pv_done[i], 1);
        }
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
    // Register split (warpgroup granularity): the producer/MMA warpgroup gives
    // registers to the two softmax warpgroups, whose threads keep a whole row
    // of S (128 values) in registers. 128 x kRegsOther + 256 x kRegsSoftmax
    // must not exceed the 384 x (registers at launch) the CTA was given; the
    // host checks the launch count before every launch.
    if (warp < 4) {
        setmaxnreg_dec<kFwdRegsOther>();
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int k_issued = 0, v_issued = 0, nq = 0;  // K/V tiles and Q pairs issued so far
            bool ok = true;
            for (int rnd = 0; ok; ++rnd) {
                const int u = fwd_unit_index(rnd, cta, G);
                if (u >= args.n_units) break;
                const FwdUnit w = fwd_unit<MASK, VARLEN>(u, args);
                // Every sequence has exactly one unit with q0 = 0 of head 0: its lengths
                // are checked against the max_seqlen bounds there.
                if (VARLEN && w.q0 == 0 && w.h == 0)
                    check_seqlens(args.cu_q, args.cu_k, w.bidx, args.Nq, args.Nk, args.err);
                if (!w.rows || w.n_kv == 0) continue;
                // Q of this unit once the previous unit's last S product has read Q.
                if (!(ok = mbar_wait(q_empty, (nq & 1) ^ 1u, wc, 60))) break;
                mbar_arrive_expect_tx(q_full, 2 * C::kTileBytes);
#pragma unroll
                for (int t = 0; t < 2; ++t)
#pragma unroll
                    for (int s = 0; s < C::kSlabs; ++s)
                        tma_load_4d(sQ + t * C::kTileBytes + s * C::kSlabBytes, &tm_q, q_full, s * C::kSlabElems, w.h,
                                    w.q_row0 + w.q0 + 128 * t, w.tma_b);
                ++nq;
                const int hk = w.h / args.group;
                for (int j = 0; j < w.n_kv; ++j) {
                    const int g = k_issued, st = g % S;
                    const uint32_t ph = (g / S) & 1;
                    if (!(ok = mbar_wait(&k_empty[st], ph ^ 1u, wc, 61))) break;
                    mbar_arrive_expect_tx(&k_full[st], C::kTileBytes);
#pragma unroll
                    for (int s = 0; s < C::kSlabs; ++s)
                        tma_load_4d(sK + st * C::kTileBytes + s * C::kSlabBytes, &tm_k, &k_full[st], s * C::kSlabElems, hk,
                                    w.k_row0 + fwd_tile<MASK>(w, j) * 128, w.tma_b);
                    ++k_issued;
                    if (!(ok = mbar_wait(&v_empty[st], ph ^ 1u, wc, 62))) break;
                    mbar_arrive_expect_tx(&v_full[st], C::kTileBytes);
#pragma unroll
                    for (int s = 0; s < C::kSlabs; ++s)
                        tma_load_4d(sV + st * C::kTileBytes + s * C::kSlabBytes, &tm_v, &v_full[st], s * C::kSlabElems, hk,
                                    w.k_row0 + fwd_tile<MASK>(w, j) * 128, w.tma_b);
                    ++v_issued;
                }
            }
            // Leave no load in flight: wait for the last one issued into every buffer.
            if (nq > 0) mbar_wait_drain(q_full, (nq - 1) & 1);
            for (int st = 0; st < S; ++st) {
                if (k_issued > st) mbar_wait_drain(&k_full[st], ((st + S * ((k_issued - 1 - st) / S)) / S) & 1);
                if (v_issued > st) mbar_wait_drain(&v_full[st], ((st + S * ((v_issued - 1 - st) / S)) / S) & 1);
            }
        }
    } else if (!C::kSepP && warp == 1) {
        // ------------------------------------------------------------ MMA issuer (d = 128)
        // One thread issues the products of both query tiles, in the order of the warp
        // roles above: each tile's batch of products runs on the tensor core without the
        // other tile's in between, so each tile's S is ready as early as it can be.
        if (lane == 0) {
            constexpr uint32_t id_qk = FP8 ? idesc_e4m3(128, 128, false, false) : idesc_f16(128, 128, BF16, false, false);
            constexpr uint32_t id_pv = FP8 ? idesc_e4m3(128, D, false, true) : idesc_f16(128, D, BF16, false, true);
            const uint32_t q_addr = smem_u32(sQ);
            // S_t = Q_t K^T with the K tile of global ring index g.
            // Descriptors of the first Q tile and of the first K / V ring slot, made once:
            // the other tiles and slots sit kTileBytes apart, and the products step through
            // an operand, by adding to the descriptor's low word.
            const SDesc qdesc = sdesc_sw128_split(q_addr, 16, 1024);
            const SDesc kdesc = sdesc_sw128_split(smem_u32(sK), 16, 1024);
            const SDesc vdesc = sdesc_sw128_split(smem_u32(sV), C::kSlabBytes, 1024);
            constexpr uint32_t kTileStep = C::kTileBytes >> 4;
            auto issue_s = [&](int t, int g) {
                const uint32_t qoff = t * kTileStep, koff = (g % S) * kTileStep;
#pragma unroll
                for (int kk = 0; kk < C::kKSteps; ++kk) {
                    const uint32_t step = ((kk >> 2) * C::kSlabBytes + (kk & 3) * 32) >> 4;
                    if constexpr (FP8)
                        mma_ss_f8(tmem + C::kColS + 128 * t,
                                  (static_cast<uint64_t>(qdesc.hi) << 32) | (qdesc.lo + qoff + step),
                                  (static_cast<uint64_t>(kdesc.hi) << 32) | (kdesc.lo + koff + step), id_qk,
                                  kk > 0 ? 1u : 0u);
                    else
                        mma_ss_split(tmem + C::kColS + 128 * t, qdesc, qoff + step, kdesc, koff + step, id_qk,
                                     kk > 0 ? 1u : 0u);
                }
                tc_commit(&s_full[t]);
            };
            int gk = 0, nq = 0;
            int ps[2] = {0, 0};  // p_full phases consumed per tile
            bool ok = true;
            for (int rnd = 0; ok; ++rnd) {
                const int u = fwd_unit_index(rnd, cta, G);
                if (u >= args.n_units) break;
                const FwdUnit w = fwd_unit<MASK, VARLEN>(u, args);
                if (!w.rows || w.n_kv == 0) continue;
                if (!(ok = mbar_wait(q_ready, nq & 1, wc, 63))) break;
                if (!(ok = mbar_wait(&k_full[gk % S], (gk / S) & 1, wc, 64))) break;
                tc_fence_after();
                // The first S products of this unit run while the softmax warpgroups
                // still write the previous unit's O (they touch only the S columns).
                for (int t = 0; t < 2; ++t)
                    if (MASK == kMaskAnchor ? fwd_active<MASK>(w, t, 0) : (w.a(t) == 0 && w.b(t) > 0)) issue_s(t, gk);
                bool started0 = false, started1 = false;  // kMaskAnchor: tile t's first P V is issued
                bool ready0 = false, ready1 = false;      // o_ready[t] committed for this unit
                if (w.n_kv == 1) tc_commit(q_empty);
                tc_commit(&k_empty[gk % S]);
                for (int j = 0; ok && j < w.n_kv; ++j) {
                    const int g = gk + j, st = g % S;
                    const bool more = j + 1 < w.n_kv;
                    if (!(ok = mbar_wait(&v_full[st], (g / S) & 1, wc, 65))) break;
                    if (more && !(ok = mbar_wait(&k_full[(g + 1) % S], ((g + 1) / S) & 1, wc, 66))) break;
                    const uint32_t v_addr = smem_u32(sV + st * C::kTileBytes);
                    // For each tile: O_t += P_t V_j, then S_t of the next key tile into the
                    // same columns. tcgen05.mma operations of one thread execute in issue
                    // order, so the second cannot overwrite P_t before the first has read
                    // it, and S_t complete implies every earlier P_t V complete.
                    for (int t = 0; ok && t < 2; ++t) {
                        // O_t is overwritten by the unit's first P_t V: the previous
                        // unit's epilogue must have read it (waited for every tile, so
                        // the phases of o_free stay in step with the units).
                        if (j == 0 && nq > 0 && !(ok = mbar_wait(&o_free[t], (nq - 1) & 1, wc, 67))) break;
                        if (!fwd_active<MASK>(w, t, j)) {
                            // under a window a tile can start later than the unit's first key
                            // tile (with anchors: again after the anchor tiles)
                            if (MASK == kMaskAnchor ? (more && fwd_active<MASK>(w, t, j + 1)) : (j + 1 == w.a(t)))
                                issue_s(t, g + 1);
                            continue;
                        }
                        if (!(ok = mbar_wait(&p_full[t], ps[t] & 1, wc, 68))) break;
                        ++ps[t];
                        tc_fence_after();
                        // O_t accumulates from the tile's second P V on.
                        const bool acc0 = MASK == kMaskAnchor ? (t ? started1 : started0) : (j > w.a(t));
                        if (t) started1 = true; else started0 = true;
                        if constexpr (FP8) {
                            // P: four E4M3 keys per column, 32 keys (8 columns, 32 rows of V)
                            // per instruction; V's d = 128 one-byte values are one 128-byte slab.
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_ts_f8(tmem + C::kColO + D * t, tmem + C::kColS + 128 * t + kk * 8,
                                          sdesc_sw128(v_addr + kk * 4096, C::kSlabBytes, 1024), id_pv,
                                          (acc0 || kk > 0) ? 1u : 0u);
                        } else {
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                mma_ts_split(tmem + C::kColO + D * t, tmem + C::kColS + 128 * t + kk * 8, vdesc,
                                             st * kTileStep + kk * 128, id_pv, (acc0 || kk > 0) ? 1u : 0u);
                        }
                        if (MASK == kMaskAnchor ? (more && fwd_active<MASK>(w, t, j + 1)) : (j + 1 < w.b(t))) {
                            issue_s(t, g + 1);
                        } else if (MASK != kMaskAnchor) {
                            // tile t's last P V of the unit: its epilogue need not wait for the
                            // other tile's last softmax and P V
                            tc_commit(&o_ready[t]);
                            if (t) ready1 = true; else ready0 = true;
                        }
                    }
                    if (j + 2 == w.n_kv) tc_commit(q_empty);  // the unit's last S products are issued
                    tc_commit(&v_empty[st]);
                    if (more) tc_commit(&k_empty[(g + 1) % S]);
                }
                if (!ready0) tc_commit(&o_ready[0]);
                if (!ready1) tc_commit(&o_ready[1]);
                gk += w.n_kv;
                ++nq;
            }
            tc_commit(mma_done);
            mbar_wait_drain(mma_done, 0);
            // TMEM is freed once the softmax warpgroups are done with it. Their waits
            // are bounded, so the arrivals come (4 s bound here as a last resort).
            const uint32_t a = smem_u32(sm_done);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < 4000000000ull) {
            }
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    } else if (C::kSepP && (warp == 1 || warp == 2)) {
        // ------------------------------------------------------------ MMA issuers (d = 64)
        // Warp 1 issues every product of query tile 0, warp 2 every product of tile 1
        // (they write disjoint TMEM columns), so each thread issues half the products of a
        // step, on its own SM sub-partition. Q and the K / V ring slots they share are
        // released by barriers that count both threads' commits. (At d = 64 each S is
        // issued as soon as its columns are free, well before the softmax needs it, so
        // the two threads' products interleaving on the tensor core costs nothing; at
        // d = 128 it delays each tile's S and the single issuer above is faster.)
        const int t = warp - 1;
        if (lane == 0) {
            constexpr uint32_t id_qk = FP8 ? idesc_e4m3(128, 128, false, false) : idesc_f16(128, 128, BF16, false, false);
            constexpr uint32_t id_pv = FP8 ? idesc_e4m3(128, D, false, true) : idesc_f16(128, D, BF16, false, true);
            // Descriptors of this thread's Q tile and of the first K / V ring slot, made once:
            // the other slots sit kTileBytes apart, and the products step through an operand,
            // by adding to the descriptor's low word.
            constexpr uint32_t kTileStep = C::kTileBytes >> 4;
            const SDesc qdesc = sdesc_sw128_split(smem_u32(sQ + t * C::kTileBytes), 16, 1024);
            const SDesc kdesc = sdesc_sw128_split(smem_u32(sK), 16, 1024);
            const SDesc vdesc = sdesc_sw128_split(smem_u32(sV), C::kSlabBytes, 1024);
            const uint32_t s_col = tmem + C::kColS + 128 * t;
            const uint32_t o_col = tmem + C::kColO + D * t;
            // S_t = Q_t K^T with the K tile of global ring index g.
            auto issue_s = [&](int g) {
                const uint32_t koff = (g % S) * kTileStep;
#pragma unroll
                for (int kk = 0; kk < C::kKSteps; ++kk) {
                    const uint32_t step = ((kk >> 2) * C::kSlabBytes + (kk & 3) * 32) >> 4;
                    if constexpr (FP8)
                        mma_ss_f8(s_col, (static_cast<uint64_t>(qdesc.hi) << 32) | (qdesc.lo + step),
                                  (static_cast<uint64_t>(kdesc.hi) << 32) | (kdesc.lo + koff + step), id_qk,
                                  kk > 0 ? 1u : 0u);
                    else
                        mma_ss_split(s_col, qdesc, step, kdesc, koff + step, id_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(&s_full[t]);
            };
            // kSepP: S_t number n (n >= 1) reuses the columns of number n - 1, which the
            // softmax must have read first.
            int ns = 0;
            auto issue_s_sep = [&](int g) -> bool {
                if (ns > 0 && !mbar_wait(&s_free[t], (ns - 1) & 1, wc, 76)) return false;
                tc_fence_after();
                issue_s(g);
                ++ns;
                return true;
            };
            int gk = 0, nq = 0;
            int ps = 0;  // p_full phases consumed
            bool ok = true;
            for (int rnd = 0; ok; ++rnd) {
                const int u = fwd_unit_index(rnd, cta, G);
                if (u >= args.n_units) break;
                const FwdUnit w = fwd_unit<MASK, VARLEN>(u, args);
                if (!w.rows || w.n_kv == 0) continue;
                if (!(ok = mbar_wait(q_ready, nq & 1, wc, 63))) break;
                if (!(ok = mbar_wait(&k_full[gk % S], (gk / S) & 1, wc, 64))) break;
                tc_fence_after();
                // The first S product of this unit runs while the softmax warpgroup still
                // writes the previous unit's O (it touches only the S columns).
                if (MASK == kMaskAnchor ? fwd_active<MASK>(w, t, 0) : (w.a(t) == 0 && w.b(t) > 0)) {
                    if constexpr (C::kSepP)
                        ok = issue_s_sep(gk);
                    else
                        issue_s(gk);
                }
                if (!ok) break;
                bool started = false;  // kMaskAnchor: the tile's first P V is issued
                if (w.n_kv == 1) tc_commit(q_empty);
                tc_commit(&k_empty[gk % S]);
                if constexpr (C::kSepP) {
                    // Per key tile j: S_t(j + 1) if the tile is active at j + 1, as soon as its
                    // softmax has read S_t(j); then P_t V_j once P_t arrives.
                    for (int j = 0; ok && j < w.n_kv; ++j) {
                        const int g = gk + j, st = g % S;
                        const bool more = j + 1 < w.n_kv;
                        if (more) {
                            // (waited for even if the tile does not need it: the slot is released below)
                            if (!(ok = mbar_wait(&k_full[(g + 1) % S], ((g + 1) / S) & 1, wc, 66))) break;
                            const bool need = MASK == kMaskAnchor ? fwd_active<MASK>(w, t, j + 1)
                                                                  : (j + 1 >= w.a(t) && j + 1 < w.b(t));
                            if (need && !(ok = issue_s_sep(g + 1))) break;
                            tc_commit(&k_empty[(g + 1) % S]);
                            if (j + 2 == w.n_kv) tc_commit(q_empty);  // the unit's last S products are issued
                        }
                        if (!(ok = mbar_wait(&v_full[st], (g / S) & 1, wc, 65))) break;
                        if (j == 0 && nq > 0 && !(ok = mbar_wait(&o_free[t], (nq - 1) & 1, wc, 67))) break;
                        if (fwd_active<MASK>(w, t, j)) {
                            if (!(ok = mbar_wait(&p_full[t], ps & 1, wc, 68))) break;
                            ++ps;
                            tc_fence_after();
                            const bool acc0 = MASK == kMaskAnchor ? started : (j > w.a(t));
                            started = true;
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                mma_ts_split(o_col, tmem + C::kColP + 64 * t + kk * 8, vdesc,
                                             st * kTileStep + kk * 128, id_pv, (acc0 || kk > 0) ? 1u : 0u);
                            tc_commit(&pv_done[t]);
                        }
                        tc_commit(&v_empty[st]);
                    }
                }
                tc_commit(&o_ready[t]);
                gk += w.n_kv;
                ++nq;
            }
            tc_commit(mma_done);
            if (t == 0) {
                // TMEM is freed once both issuers' products are complete and the softmax
                // warpgroups are done with it. Every wait is bounded, so the arrivals come
                // (4 s bounds here as a last resort).
                for (uint64_t* bar : {mma_done, sm_done}) {
                    const uint32_t a = smem_u32(bar);
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < 4000000000ull) {
                    }
                }
            }
        }
        __syncwarp();
        if (t == 0) {
            tc_fence_after();
            tmem_dealloc(tmem, C::kTmemCols);
        }
    }
        return;  // warps 0-3 end here; no code is shared with the softmax warpgroups
    } else {
        setmaxnreg_inc<kFwdRegsSoftmax>();
        // ------------------------------------------------------------ softmax / correction / epilogue
        const int t = (warp - 4) >> 2;  // query tile of this warpgroup
        const int w4 = warp & 3;
        const int r = w4 * 32 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(w4 * 32) << 16);
        const uint32_t s_addr = lane_base + C::kColS + 128 * t;
        const uint32_t o_addr = lane_base + C::kColO + D * t;
        const uint32_t p_addr = lane_base + C::kColP + 64 * t;  // kSepP
        const float sl2_base = args.scale_log2;
        int ss = 0, nq = 0;  // s_full phases consumed; units with work done
        int np = 0;          // kSepP: P_t written so far (each followed by one P_t V)
        bool ok = true;
        for (int rnd = 0; ok; ++rnd) {
            const int u = fwd_unit_index(rnd, cta, G);
            if (u >= args.n_units) break;
            const FwdUnit w = fwd_unit<MASK, VARLEN>(u, args);
            if (!w.rows) continue;
            const int qt0 = w.q0 + 128 * t;
            const int q = qt0 + r;
            const int nt = fwd_tile_steps<MASK>(w, t);  // key tiles fwd_tile_of(w, t, jj), jj < nt
            // This thread's output row (computed where it is used, to keep registers
            // free during the key loop).
            // (The unit is decoded again there: nothing of it stays live across the loop.)
            auto row_ok = [&](const FwdUnit& x) -> bool {
                if constexpr (VARLEN) return q < x.q_len && x.q_row0 + q >= 0 && x.q_row0 + q < args.total_q;
                return q < x.q_len;
            };
            auto out_row = [&](const FwdUnit& x) -> T16* {
                const long long row = VARLEN ? static_cast<long long>(x.q_row0 + q) * args.o_ss
                                             : x.bidx * args.o_sb + static_cast<long long>(q) * args.o_ss;
                return o_base + row + x.h * args.o_sh;
            };
            auto lse_row = [&](const FwdUnit& x) -> float* {
                return VARLEN ? args.lse + static_cast<size_t>(x.h) * args.total_q + x.q_row0 + q
                              : args.lse + (static_cast<size_t>(x.bidx) * args.Hq + x.h) * args.Nq + q;
            };
            if (w.n_kv == 0) {  // no row of this unit sees any key: O = 0, L = -inf
                if (row_ok(w)) {
                    uint4* d4 = reinterpret_cast<uint4*>(out_row(w));
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) d4[c] = make_uint4(0, 0, 0, 0);
                    *lse_row(w) = -INFINITY;
                }
                continue;
            }
            // This row's visible keys, relative to the first key of this warpgroup's
            // first step: [rel_lo, rel_hi).
            int rel_lo, rel_hi;
            key_range<MASK>(args, q, w.q_len, w.k_len, rel_lo, rel_hi);
            const int key_lo = rel_lo, key_hi = rel_hi;  // kMaskAnchor: absolute bounds
            rel_lo -= (w.jlo + w.a(t)) * 128;
            rel_hi -= (w.jlo + w.a(t)) * 128;
            if constexpr (QKNORM) {  // this thread's row of Q, before the unit's first S product
                ok = warp_all(mbar_wait(q_full, nq & 1, wc, 57));
                if (!ok) break;
                rms_normalise_row<D, BF16>(sQ + t * C::kTileBytes, r, args.norm_eps);
                fence_proxy_async_smem();
                mbar_arrive(q_norm);
            }
            // FP8: the query tile's dequantisation factor, and V's largest block factor
            // over the tiles this warpgroup visits (P carries v_j / v_max <= 1).
            float fq = 1.f, v_max = 1.f;
            const float* ksc = nullptr;
            const float* vsc = nullptr;
            if constexpr (FP8) {
                const int hkv = w.h / args.group;
                const size_t kv_row = (static_cast<size_t>(w.bidx) * (args.Hq / args.group) + hkv) * args.nkb;
                fq = args.q_scale[(static_cast<size_t>(w.bidx) * args.Hq + w.h) * args.nqb +
                                  min(qt0 >> 7, args.nqb - 1)];
                ksc = args.k_scale + kv_row + w.jlo + w.a(t);
                vsc = args.v_scale + kv_row + w.jlo + w.a(t);
                v_max = 0.f;
                for (int jj = 0; jj < nt; ++jj) v_max = fmaxf(v_max, vsc[jj]);
            }
            float m = -INFINITY, l = 0.f, lr = 0.f;
            for (int j = 0; j < nt; ++j) {
                // Exp2 factor of this (query tile, key tile) pair; with FP8 also P's factor
                // v_j / v_max as a bias in the exponent, and v_max / v_j back for l.
                float sl2 = sl2_base, bias = 0.f, vr = 1.f;
                if constexpr (FP8) {
                    sl2 = sl2_base * fq * ksc[j];
                    const float vj = vsc[j];
                    vr = v_max / vj;
                    float lg;
                    asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(vj / v_max));
                    bias = lg;
                }
                ok = warp_all(mbar_wait(&s_full[t], ss & 1, wc, 69));
                if (!ok) break;
                ++ss;
                tc_fence_after();
                // Columns >= lim are masked, and under a window columns < lim_lo (with
                // anchors only those at or past anc, the first key that is not an anchor).
                const int kb = MASK == kMaskAnchor ? fwd_tile_of<MASK>(w, t, j) * 128 : 0;
                const int lim = MASK == kMaskAnchor ? key_hi - kb : rel_hi - j * 128;
                const int lim_lo = MASK == kMaskAnchor ? key_lo - kb : rel_lo - j * 128;
                const int anc = args.n_anchor - kb;
                // Key mask: the keep bits of this key tile's 128 keys (all set: nothing to do).
                uint32_t kw0 = ~0u, kw1 = ~0u, kw2 = ~0u, kw3 = ~0u;
                if constexpr (KEYMASK) {
                    const int ktile = fwd_tile_of<MASK>(w, t, j);
                    const uint32_t* kbp = args.key_bits + static_cast<size_t>(w.bidx) * args.kb_words + ktile * 4;
                    const int rem = args.kb_words - ktile * 4;
                    kw0 = rem > 0 ? kbp[0] : 0u;
                    kw1 = rem > 1 ? kbp[1] : 0u;
                    kw2 = rem > 2 ? kbp[2] : 0u;
                    kw3 = rem > 3 ? kbp[3] : 0u;
                }
                const bool keys_masked = KEYMASK && (kw0 & kw1 & kw2 & kw3) != ~0u;
                // (uniform per warp: only tiles on a window's edge pay for the mask)
                const bool need_mask =
                    __any_sync(0xffffffffu, lim < 128 || (MASK == kMaskWindow && lim_lo > 0) ||
                                                (MASK == kMaskAnchor && lim_lo > 0 && lim_lo > anc) || keys_masked);
                uint32_t sv[4][32];
    #pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + 32 * c, sv[c]);
    #pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld_wait(sv[c]);
                if constexpr (C::kSepP) {  // S_t is in registers: its columns may take the next S_t
                    tc_fence_before();
                    mbar_arrive(&s_free[t]);
                }
                if (need_mask) {  // masked columns read as -inf: out of the max, P = 0
    #pragma unroll
                    for (int c = 0; c < 128; ++c) {
                        const uint32_t kw = c < 32 ? kw0 : (c < 64 ? kw1 : (c < 96 ? kw2 : kw3));
                        if (c >= lim || (MASK == kMaskWindow && c < lim_lo) ||
                            (MASK == kMaskAnchor && c < lim_lo && c >= anc) || (KEYMASK && !((kw >> (c & 31)) & 1u)))
                            sv[c >> 5][c & 31] = __float_as_uint(-INFINITY);
                    }
                }
                // Row max: 8 independent chains of three-input max.
                float mxp[8];
    #pragma unroll
                for (int i = 0; i < 8; ++i) mxp[i] = -INFINITY;
    #pragma unroll
                for (int i = 0; i < 64; ++i)
                    mxp[i & 7] = fmax3(mxp[i & 7], __uint_as_float(sv[(2 * i) >> 5][(2 * i) & 31]),
                                       __uint_as_float(sv[(2 * i + 1) >> 5][(2 * i + 1) & 31]));
                const float mx = fmax3(fmax3(mxp[0], mxp[1], mxp[2]), fmax3(mxp[3], mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7]));
                const float m_new = fmaxf(m, mx * sl2);
                float alpha = 1.f;
                bool resc = false;
                if (m_new > m + kRescaleThreshold) {  // false while the row has seen no key
                    if (m != -INFINITY) {
                        alpha = ex2_approx(m - m_new);
                        resc = true;
                    }
                    m = m_new;
                }
                const float neg_m = (m == -INFINITY) ? 0.f : -m;
                // P = 2^(S c - m) as 16-bit pairs (keys 2i, 2i + 1 in column i), partial sums
                // of the exact and of the rounded values.
                // Pairs of keys go through the packed f32x2 FMA and adds.
                const uint64_t c2 = f2_pack(sl2, sl2), m2 = f2_pack(neg_m + bias, neg_m + bias);
                uint64_t rs2[4] = {0, 0, 0, 0}, rsr2[4] = {0, 0, 0, 0};  // (0.f, 0.f) pairs
                if constexpr (FP8) {
                    // Four E4M3 keys per column (4i .. 4i + 3 in column i, the lowest in the
                    // low byte); O is normalised by the exact sum.
                    uint32_t pk8[32];
    #pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const uint64_t xa = f2_pack(__uint_as_float(sv[(4 * i) >> 5][(4 * i) & 31]),
                                                    __uint_as_float(sv[(4 * i + 1) >> 5][(4 * i + 1) & 31]));
                        const uint64_t xb = f2_pack(__uint_as_float(sv[(4 * i + 2) >> 5][(4 * i + 2) & 31]),
                                                    __uint_as_float(sv[(4 * i + 3) >> 5][(4 * i + 3) & 31]));
                        float y0, y1, y2, y3;
                        f2_unpack(f2_fma(xa, c2, m2), y0, y1);
                        f2_unpack(f2_fma(xb, c2, m2), y2, y3);
                        const float p0 = ex2_approx(y0), p1 = ex2_approx(y1);
                        const float p2 = ex2_approx(y2), p3 = ex2_approx(y3);
                        rs2[i & 3] = f2_add(rs2[i & 3], f2_add(f2_pack(p0, p1), f2_pack(p2, p3)));
                        pk8[i] = pack4_e4m3(p0, p1, p2, p3);
                    }
                    tmem_st32(s_addr + 0, pk8);
                } else {
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
                    if constexpr (C::kSepP) {
                        // P_t's columns and O_t are free once the previous P_t V is complete.
                        if (np > 0) {
                            ok = warp_all(mbar_wait(&pv_done[t], (np - 1) & 1, wc, 77));
                            if (!ok) break;
                        }
                        ++np;
                        tc_fence_after();
                        tmem_st32(p_addr + 0, pk[0]);
                        tmem_st32(p_addr + 32, pk[1]);
                    } else {
                        tmem_st32(s_addr + 0, pk[0]);
                        tmem_st32(s_addr + 32, pk[1]);
                    }
                }
                const float rs = f2_sum(f2_add(f2_add(rs2[0], rs2[1]), f2_add(rs2[2], rs2[3])));
                const float rsr = f2_sum(f2_add(f2_add(rsr2[0], rsr2[1]), f2_add(rsr2[2], rsr2[3])));
                l = l * alpha + rs * vr;
                lr = lr * alpha + rsr;
                // S_t was issued after the previous key tile's P_t V and MMAs of one thread
                // complete in order, so O_t is final for that tile here and can be
                // rescaled in place (kSepP: pv_done was waited for above).
                if (j > 0 && __any_sync(0xffffffffu, resc)) {
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
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&p_full[t]);
            }
            if (!ok) break;
            // (decoded again while the last P V runs)
            const FwdUnit we = fwd_unit<MASK, VARLEN>(u, args);
            const bool out_ok = row_ok(we);
            T16* dst = out_ok ? out_row(we) : nullptr;
            const float inv_l = FP8 ? (l > 0.f ? v_max / l : 0.f) : ((lr > 0.f) ? 1.f / lr : 0.f);
            ok = warp_all(mbar_wait(&o_ready[t], nq & 1, wc, 70));
            if (!ok) break;
            ++nq;
            tc_fence_after();
            // O leaves through the warp's staging buffer, one 32-column chunk (64 bytes
            // a row) at a time: each thread writes its row's chunk, then lane i stores
            // bytes 16 (i % 4) .. + 16 of row 8 k + i / 4 (k = 0 .. 3), so one store
            // instruction covers eight 64-byte row segments instead of 32 scattered 16-byte
            // pieces. The 16-byte pieces are XOR-swizzled by row pair: both the row-wise
            // writes and the segment-wise reads then touch each bank group once per
            // quarter warp.
            const uint32_t stg = smem_u32(sEpi + (warp - 4) * C::kEpiBytesPerWarp);
            const int piece = lane & 3;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t pk[16];
                if (nt > 0) {
                    uint32_t ov[32];
                    tmem_ld32(o_addr + c0, ov);
                    tmem_ld_wait(ov);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = pack2<BF16>(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = 0u;
                }
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    st_shared_v4(stg + lane * 64 + ((p ^ ((lane >> 1) & 3)) << 4), pk[4 * p], pk[4 * p + 1],
                                 pk[4 * p + 2], pk[4 * p + 3]);
                __syncwarp();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int rr = 8 * k + (lane >> 2);
                    const uint4 val = ld_shared_v4(stg + rr * 64 + ((piece ^ ((rr >> 1) & 3)) << 4));
                    // row rr's address and validity, from the thread that owns the row
                    const bool seg_ok = __shfl_sync(0xffffffffu, out_ok, rr);
                    T16* seg = reinterpret_cast<T16*>(
                        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(dst), rr));
                    if (seg_ok) *reinterpret_cast<uint4*>(seg + c0 + 8 * piece) = val;
                }
                __syncwarp();
            }
            // O_t's columns are free for the next unit's first P_t V.
            tc_fence_before();
            mbar_arrive(&o_free[t]);
            if (out_ok) {
                float L = -INFINITY;
                if (l > 0.f) {
                    float lg;
                    asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(l));
                    L = (m + lg) * kLn2;
                }
                *lse_row(we) = L;
            }
        }
        tc_fence_before();
        mbar_arrive(sm_done);
    }
}

// RMS normalisation of rows of d 16-bit values (unit gain, fp32 arithmetic, rounded
// to the 16-bit type): d / 8 threads per row, 8 values each.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_rms_normalise_rows(const uint16_t* x, uint16_t* y, size_t rows, float eps) {
    constexpr int kLanes = D / 8;
    const size_t row = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) / kLanes;
    const int sub = threadIdx.x % kLanes;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (row < rows) v = reinterpret_cast<const uint4*>(x + row * D)[sub];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint64_t acc = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint64_t p = f2_pack(unpack_lo<BF16>(w[i]), unpack_hi<BF16>(w[i]));
        acc = f2_fma(p, p, acc);
    }
    float ss = f2_sum(acc);
#pragma unroll
    for (int off = kLanes / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = rsqrtf(ss * (1.f / D) + eps);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = pack2<BF16>(unpack_lo<BF16>(w[i]) * inv, unpack_hi<BF16>(w[i]) * inv);
    if (row < rows) reinterpret_cast<uint4*>(y + row * D)[sub] = make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace fa
