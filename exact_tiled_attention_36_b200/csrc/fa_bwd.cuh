// fa_bwd.cuh: tiled exact attention backward for sm_100a.
//
// The backward recomputes S and P from the saved log-sum-exp L and dO, so no
// N x N matrix is stored ("FlashAttention/zh", section "backward pass and
// recomputation"). With P = exp(scale Q K^T - L) the kernels compute the exact
// gradient of the definition:
//     D_i = sum_c dO_ic O_ic           (equals sum_j P_ij dP_ij)
//     dP = dO V^T,  dS = P o (dP - D),  dV = P^T dO,
//     dK = scale dS^T Q,  dQ = scale dS K,
// and with grouped KV heads dK, dV of a KV head sum over its query heads.
//
// Three kernels run in order on the caller's stream:
//   fa_bwd_preprocess  D = rowsum(dO o O) (fp32) and dQ_acc = 0.
//   fa_bwd_kernel      one CTA per (128-key tile j, KV head, batch). K_j and V_j
//                      stay in shared memory; for every query head of the
//                      group and every 128-query tile i it recomputes
//                        S^T = K_j Q_i^T and dP^T = V_j dO_i^T   (TMEM, fp32)
//                      turns them into P^T and dS^T (16-bit, written back over
//                      the same TMEM columns, dS also to shared memory), then
//                        dV += P^T dO_i,  dK += dS^T Q_i          (TMEM, fp32)
//                        dQ_i = dS K_j                             (TMEM, fp32)
//                      and adds dQ_i into the fp32 accumulator with vector
//                      reductions. dK, dV leave TMEM once, at the end.
//   fa_bwd_dq_convert  dQ = dtype(scale * dQ_acc).
//   (d = 128 runs fa_bwd128_kernel of fa_bwd128.cuh in place of fa_bwd_kernel
//   and fa_bwd_dq_convert_g4 in place of fa_bwd_dq_convert.)
//
// Warp roles of fa_bwd_kernel (384 threads): warp 0 TMA producer, warp 1 TMEM
// allocation and the single MMA-issuing thread, warps 2-3 idle, warps 4-11 two
// compute warpgroups (each owns half of the 128 query columns of S^T / dP^T,
// half of the dQ columns while draining, and one of dV / dK at the end).
//
// TMEM columns: [0,128) S^T, later P^T, later dQ_i; [128,256) dP^T, later dS^T;
// [256,256+d) dV; [256+d,256+2d) dK. Each compute warpgroup writes its packed
// 16-bit P^T / dS^T over the first half of its own 64 columns.
#pragma once

#include <cuda_fp16.h>

#include "sm100.cuh"

namespace fa {

struct BwdArgs {
    const float* lse;  // [B, Hq, Nq]
    const float* D;    // [B, Hq, Nq]
    float* dq_acc;     // d = 64: [B, Nq, Hq, 64]; d = 128: [B, Hq, nq4, 128, 4] (see fa_bwd_dq_convert_g4)
    int nq4;           // groups of four queries per (b, h) in the d = 128 layout: ceil(Nq / 4)
    void* dk;          // [B, Nk, Hkv, d]
    void* dv;
    int Hq, Hkv, group, Nq, Nk;  // varlen: Nq, Nk are the max_seqlen bounds
    const int* cu_q;             // varlen: [num_seqs + 1] row offsets of the packed buffers
    const int* cu_k;
    int total_q;                 // varlen: rows of q / o / dO (L and D are [Hq, total_q])
    float scale;
    float scale_log2;
    int wl, wr;  // MASKED: keys from wl before to wr after the aligned diagonal (< 0: unbounded)
    int n_anchor;  // MASKED: keys 0 .. n_anchor - 1 are also visible below the window (global anchors)
    // dK and dV element strides: batch, token, head (d contiguous); varlen uses token
    // (the packed row) and head only.
    long long dk_sb, dk_ss, dk_sh, dv_sb, dv_ss, dv_sh;
    // Key mask (null: none): bit j % 32 of word b * kb_words + j / 32 set = key j of batch b
    // is visible (ANDed with the window).
    const uint32_t* key_bits;
    int kb_words;
    // d = 128 under the causal mask: 1 = the grid is (key tiles, Hkv, sequences), every key
    // tile of a (sequence, KV head) dispatched together; 0 = (Hkv, sequences, key tiles),
    // the first key tiles of every pair first (see fa_bwd128_kernel).
    int kt_fast;
    int* err;
};

// Key `key` of batch b is visible under the key mask of `a` (always without one).
__device__ __forceinline__ bool key_kept(const BwdArgs& a, int b, int key) {
    return a.key_bits == nullptr ||
           ((a.key_bits[static_cast<size_t>(b) * a.kb_words + (key >> 5)] >> (key & 31)) & 1u) != 0u;
}

// Some key of the tile [k0, min(k0 + 128, Nk)) of batch b is masked out by the key mask.
__device__ __forceinline__ bool tile_keys_masked(const BwdArgs& a, int b, int k0, int Nk) {
    if (a.key_bits == nullptr) return false;
    bool masked = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int kw = k0 + 32 * i;  // first key of word i
        if (kw >= Nk) break;
        const uint32_t valid = Nk - kw >= 32 ? ~0u : ((1u << (Nk - kw)) - 1u);
        const uint32_t w = a.key_bits[static_cast<size_t>(b) * a.kb_words + (kw >> 5)];
        masked = masked || ((w & valid) != valid);
    }
    return masked;
}

// Queries [qlo, qhi) that see key `key` (bottom-right alignment: query q's aligned
// key is q + Nk - Nq; with MASKED the window (wl, wr) of BwdArgs, else every query).
// An anchor key (key < n_anchor) is seen by every query its right bound allows.
template <bool MASKED>
__device__ __forceinline__ void query_range(const BwdArgs& a, int key, int Nq, int Nk, int& qlo, int& qhi) {
    qlo = 0;
    qhi = Nq;
    if (MASKED) {
        const int q_aligned = key - (Nk - Nq);
        if (a.wr >= 0) qlo = max(0, q_aligned - a.wr);
        if (a.wl >= 0 && key >= a.n_anchor) qhi = min(Nq, q_aligned + a.wl + 1);
    }
}

// Query tiles [i0, i0 + n_i) that see some key of the key tile at k0.
template <bool MASKED>
__device__ __forceinline__ void query_tiles(const BwdArgs& a, int k0, int Nq, int Nk, int& i0, int& n_i) {
    int qlo, qhi, qlo2, qhi2;
    query_range<MASKED>(a, k0, Nq, Nk, qlo, qhi);
    query_range<MASKED>(a, min(k0 + 127, Nk - 1), Nq, Nk, qlo2, qhi2);
    qhi2 = max(qhi, qhi2);  // an anchor first key sees further than the tile's last key
    i0 = qlo / 128;
    const int i_end = qhi2 > qlo ? (qhi2 + 127) / 128 : i0;
    n_i = i_end - i0;
}

template <int D>
struct BwdCfg {
    static constexpr int kSlabBytes = 128 * 128;
    static constexpr int kTileBytes = (D / 64) * kSlabBytes;  // 128 rows x d, 16-bit
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kKOff + kTileBytes;
    static constexpr int kQOff = kVOff + kTileBytes;     // 2 stages
    static constexpr int kDOOff = kQOff + 2 * kTileBytes;  // 2 stages
    static constexpr int kDSOff = kDOOff + 2 * kTileBytes;  // dS [128 q x 128 keys], MN-major for the dQ MMA
    static constexpr int kLDOff = kDSOff + 2 * kSlabBytes;  // 2 stages of L*log2e [128] and D [128], fp32
    static constexpr int kBarOff = kLDOff + 2048;
    static constexpr int kNumBars = 1 + 2 + 2 + 1 + 1 + 1 + 1 + 1 + 1 + 2;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

constexpr int kBwdThreads = 384;

template <int D, bool BF16, bool CAUSAL, bool VARLEN = false>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdArgs args) {
    using C = BwdCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (!smem_base_ok(smem, args.err)) return;  // the 128-byte swizzle needs 1024-byte aligned tiles

    // Non-causal grid (key tiles, Hkv, batches); causal grid (Hkv, batches, key
    // tiles) so that the first key tiles, which see the most query tiles, are
    // dispatched first.
    const int kt = CAUSAL ? static_cast<int>(blockIdx.z) : static_cast<int>(blockIdx.x);
    const int hk = CAUSAL ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.y);
    const int b = CAUSAL ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.z);
    const int k0 = kt * 128;
    // Rows of this sequence: fixed length, or varlen (b is the sequence; its rows
    // start at q_row0 / k_row0 of the packed buffers, and the rows of a tile past its
    // lengths belong to the next sequence, so they are masked, not zero-filled).
    int q_len, k_len, q_row0, k_row0, tma_b;
    if constexpr (VARLEN) {
        q_row0 = args.cu_q[b];
        k_row0 = args.cu_k[b];
        q_len = min(args.cu_q[b + 1] - q_row0, args.Nq);
        k_len = min(args.cu_k[b + 1] - k_row0, args.Nk);
        tma_b = 0;
        // one CTA per sequence checks its lengths against the max_seqlen bounds
        if (kt == 0 && hk == 0 && threadIdx.x == 0)
            check_seqlens(args.cu_q, args.cu_k, b, args.Nq, args.Nk, args.err);
        if (k0 >= k_len) return;  // the tile lies past this sequence's keys
    } else {
        q_row0 = 0;
        k_row0 = 0;
        q_len = args.Nq;
        k_len = args.Nk;
        tma_b = b;
    }
    const int Nq = q_len, Nk = k_len;
    // Element offsets of key `key` of this sequence in the dK and dV buffers.
    auto dk_off = [&](int key) -> long long {
        return VARLEN ? (k_row0 + key) * args.dk_ss + hk * args.dk_sh : b * args.dk_sb + key * args.dk_ss + hk * args.dk_sh;
    };
    auto dv_off = [&](int key) -> long long {
        return VARLEN ? (k_row0 + key) * args.dv_ss + hk * args.dv_sh : b * args.dv_sb + key * args.dv_ss + hk * args.dv_sh;
    };
    int i0, n_i;
    query_tiles<CAUSAL>(args, k0, Nq, Nk, i0, n_i);
    const int n_it = args.group * n_i;

    using T16 = uint16_t;
    const int warp = warp_id();
    const int lane = lane_id();

    if (n_it == 0) {  // no query sees this key tile: dK = dV = 0
        if (threadIdx.x < 128) {
            const int key = k0 + static_cast<int>(threadIdx.x);
            if (key < Nk) {
                uint4* a = reinterpret_cast<uint4*>(static_cast<T16*>(args.dk) + dk_off(key));
                uint4* c = reinterpret_cast<uint4*>(static_cast<T16*>(args.dv) + dv_off(key));
#pragma unroll
                for (int i = 0; i < D / 8; ++i) a[i] = c[i] = make_uint4(0, 0, 0, 0);
            }
        }
        return;
    }

    uint8_t* sK = smem + C::kKOff;
    uint8_t* sV = smem + C::kVOff;
    uint8_t* sQ = smem + C::kQOff;
    uint8_t* sDO = smem + C::kDOOff;
    uint8_t* sDS = smem + C::kDSOff;
    float* sLD = reinterpret_cast<float*>(smem + C::kLDOff);  // stage st: L2 at [256 st], D at [256 st + 128]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* kv_full = bars;
    uint64_t* q_full = bars + 1;   // [2]
    uint64_t* q_empty = bars + 3;  // [2]
    uint64_t* s_full = bars + 5;
    uint64_t* ds_ready = bars + 6;
    uint64_t* mm_done = bars + 7;
    uint64_t* dq_full = bars + 8;
    uint64_t* dq_free = bars + 9;
    uint64_t* fin = bars + 10;
    uint64_t* ld_full = bars + 11;  // [2]
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    int* abort_flag = reinterpret_cast<int*>(smem + C::kMiscOff + 4);

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(ds_ready, 256);
        mbar_init(mm_done, 1);
        mbar_init(dq_full, 1);
        mbar_init(dq_free, 256);
        mbar_init(fin, 1);
        mbar_init(&ld_full[0], 128);
        mbar_init(&ld_full[1], 128);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_do);
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
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_expect_tx(kv_full, 2 * C::kTileBytes);
#pragma unroll
            for (int s = 0; s < D / 64; ++s) {
                tma_load_4d(sK + s * C::kSlabBytes, &tm_k, kv_full, s * 64, hk, k_row0 + k0, tma_b);
                tma_load_4d(sV + s * C::kSlabBytes, &tm_v, kv_full, s * 64, hk, k_row0 + k0, tma_b);
            }
            int issued = 0;
            for (int it = 0; it < n_it; ++it) {
                const int st = it & 1;
                const int h = hk * args.group + it / n_i;
                const int q0 = (i0 + it % n_i) * 128;
                if (!mbar_wait(&q_empty[st], ((it >> 1) & 1) ^ 1u, wc, 21)) break;
                mbar_arrive_expect_tx(&q_full[st], 2 * C::kTileBytes);
#pragma unroll
                for (int s = 0; s < D / 64; ++s) {
                    tma_load_4d(sQ + st * C::kTileBytes + s * C::kSlabBytes, &tm_q, &q_full[st], s * 64, h,
                                q_row0 + q0, tma_b);
                    tma_load_4d(sDO + st * C::kTileBytes + s * C::kSlabBytes, &tm_do, &q_full[st], s * 64, h,
                                q_row0 + q0, tma_b);
                }
                ++issued;
            }
            mbar_wait_drain(kv_full, 0);
            for (int st = 0; st < 2; ++st)
                if (issued > st) mbar_wait_drain(&q_full[st], (((issued - 1 - st) / 2 * 2 + st) >> 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_kk = idesc_f16(128, 128, BF16, false, false);  // S^T, dP^T
            constexpr uint32_t id_tm = idesc_f16(128, D, BF16, false, true);     // dV, dK (A in TMEM)
            constexpr uint32_t id_dq = idesc_f16(128, D, BF16, true, true);      // dQ (A = dS, MN-major)
            const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV), ds_addr = smem_u32(sDS);
            bool ok = mbar_wait(kv_full, 0, wc, 22);
            for (int it = 0; ok && it < n_it; ++it) {
                const int st = it & 1;
                if (it > 0 && !(ok = mbar_wait(dq_free, (it - 1) & 1, wc, 23))) break;  // dQ_{it-1} drained
                if (!(ok = mbar_wait(&q_full[st], (it >> 1) & 1, wc, 24))) break;
                tc_fence_after();
                const uint32_t q_addr = smem_u32(sQ + st * C::kTileBytes);
                const uint32_t do_addr = smem_u32(sDO + st * C::kTileBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kSlabBytes + (kk & 3) * 32;
                    mma_ss(tmem + C::kColS, sdesc_sw128(k_addr + off, 16, 1024), sdesc_sw128(q_addr + off, 16, 1024),
                           id_kk, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kSlabBytes + (kk & 3) * 32;
                    mma_ss(tmem + C::kColDP, sdesc_sw128(v_addr + off, 16, 1024),
                           sdesc_sw128(do_addr + off, 16, 1024), id_kk, kk > 0 ? 1u : 0u);
                }
                tc_commit(s_full);
                if (!(ok = mbar_wait(ds_ready, it & 1, wc, 25))) break;
                tc_fence_after();
                // P^T / dS^T of queries 16 kk .. 16 kk + 15 sit at column
                // 64 (kk / 4) + 8 (kk % 4) of their region (see the compute warps).
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + C::kColDV, tmem + C::kColS + (kk >> 2) * 64 + (kk & 3) * 8,
                           sdesc_sw128(do_addr + kk * 2048, C::kSlabBytes, 1024), id_tm, (it > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + C::kColDK, tmem + C::kColDP + (kk >> 2) * 64 + (kk & 3) * 8,
                           sdesc_sw128(q_addr + kk * 2048, C::kSlabBytes, 1024), id_tm, (it > 0 || kk > 0) ? 1u : 0u);
                // dQ_i overwrites the P^T columns and the next dP^T the dS^T
                // columns; both are different accumulators, so wait explicitly.
                tc_commit(mm_done);
                if (!(ok = mbar_wait(mm_done, it & 1, wc, 26))) break;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tmem + C::kColS, sdesc_sw128(ds_addr + kk * 2048, C::kSlabBytes, 1024),
                           sdesc_sw128(k_addr + kk * 2048, C::kSlabBytes, 1024), id_dq, kk > 0 ? 1u : 0u);
                tc_commit(&q_empty[st]);
                tc_commit(dq_full);
            }
            tc_commit(fin);
            mbar_wait_drain(fin, 0);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ compute warpgroups
        const int wg = (warp - 4) >> 2;  // 0 or 1
        const int w4 = warp & 3;
        const int r = w4 * 32 + lane;  // TMEM lane: key row for S^T / dP^T / dV / dK, query row for dQ
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(w4 * 32) << 16);
        const int key = k0 + r;
        const bool key_in = key < Nk;                          // a row of dK / dV to write
        const bool key_ok = key_in && key_kept(args, b, key);  // a key that takes part
        const float sl2 = args.scale_log2;
        constexpr float kLog2eF = 1.4426950408889634074f;
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const int h = hk * args.group + it / n_i;
            const int q0 = (i0 + it % n_i) * 128;
            // Per-query L (in log2 units) and D of this tile, shared through a
            // 2-stage smem buffer. Stage it&1 is rewritten at it+2, when every
            // compute thread has arrived on ds_ready for it+1, so no reader of
            // iteration it is left.
            float* sL = sLD + (it & 1) * 256;
            float* sD = sL + 128;
            if (wg == 0) {
                const int q = q0 + r;
                float l2 = INFINITY, dd = 0.f;
                if (q < Nq) {
                    const size_t row = VARLEN ? static_cast<size_t>(h) * args.total_q + q_row0 + q
                                              : (static_cast<size_t>(b) * args.Hq + h) * Nq + q;
                    const float L = args.lse[row];
                    l2 = (L == -INFINITY) ? INFINITY : L * kLog2eF;  // a row that saw no key has P = 0
                    dd = args.D[row];
                }
                sL[r] = l2;
                sD[r] = dd;
                mbar_arrive(&ld_full[it & 1]);
            }
            ok = warp_all(mbar_wait(&ld_full[it & 1], (it >> 1) & 1, wc, 30));
            if (!ok) break;
            ok = warp_all(mbar_wait(s_full, it & 1, wc, 27));
            if (!ok) break;
            tc_fence_after();
            // Queries [qlim, qlim_hi) see this thread's key (and only if key < Nk).
            int qlim, qlim_hi;
            query_range<CAUSAL>(args, key, Nq, Nk, qlim, qlim_hi);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = wg * 2 + cc;  // 32-column chunk of the 128 queries
                uint32_t sv[32], pv[32];
                tmem_ld32(lane_base + C::kColS + c * 32, sv);
                tmem_ld32(lane_base + C::kColDP + c * 32, pv);
                tmem_ld_wait(sv);
                tmem_ld_wait(pv);
                uint32_t pk[16], dk16[16];
#pragma unroll
                for (int t = 0; t < 32; t += 2) {
                    float p[2], ds[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int qq = c * 32 + t + e;
                        bool vis = key_ok;
                        if (CAUSAL) vis = vis && (q0 + qq >= qlim) && (q0 + qq < qlim_hi);
                        const float pe = ex2_approx(fmaf(__uint_as_float(sv[t + e]), sl2, -sL[qq]));
                        p[e] = vis ? pe : 0.f;
                        ds[e] = p[e] * (__uint_as_float(pv[t + e]) - sD[qq]);
                    }
                    pk[t >> 1] = pack2<BF16>(p[0], p[1]);
                    dk16[t >> 1] = pack2<BF16>(ds[0], ds[1]);
                }
                // Packed 16-bit pairs go over columns this warpgroup has already
                // read itself: queries 64 wg + 32 cc + t land in column
                // 64 wg + 16 cc + t / 2 (the other warpgroup may still be reading
                // its own half).
                tmem_st16(lane_base + C::kColS + wg * 64 + cc * 16, pk);
                tmem_st16(lane_base + C::kColDP + wg * 64 + cc * 16, dk16);
                // dS row of this key into the MN-major dQ operand: 64-query slabs,
                // key rows of 128 B, 16-byte chunks swizzled by key % 8.
                uint8_t* row = sDS + (c >> 1) * C::kSlabBytes + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int chunk = ((c & 1) * 4 + u) ^ (r & 7);
                    *reinterpret_cast<uint4*>(row + chunk * 16) =
                        make_uint4(dk16[4 * u], dk16[4 * u + 1], dk16[4 * u + 2], dk16[4 * u + 3]);
                }
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(ds_ready);
            // Drain dQ_i = dS K_j: lane r is query q0 + r; this warpgroup adds d/2 columns.
            ok = warp_all(mbar_wait(dq_full, it & 1, wc, 28));
            if (!ok) break;
            tc_fence_after();
            const int q = q0 + r;
            // [sequences, max_seqlen_q, Hq, d] (fixed length: args.Nq = Nq)
            float* dst = args.dq_acc + ((static_cast<size_t>(b) * args.Nq + q) * args.Hq + h) * D;
#pragma unroll
            for (int c0 = wg * (D / 2); c0 < (wg + 1) * (D / 2); c0 += 32) {
                uint32_t v[32];
                tmem_ld32(lane_base + C::kColS + c0, v);
                tmem_ld_wait(v);
                if (q < Nq) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        red_add_v4(dst + c0 + i, __uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                   __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
                }
            }
            tc_fence_before();
            mbar_arrive(dq_free);
        }
        if (ok) ok = warp_all(mbar_wait(fin, 0, wc, 29));
        if (ok) {
            tc_fence_after();
            // Warpgroup 0 writes dV, warpgroup 1 writes dK = scale * (dS^T Q).
            const uint32_t col = wg == 0 ? C::kColDV : C::kColDK;
            const float mul = wg == 0 ? 1.f : args.scale;
            T16* dst = wg == 0 ? static_cast<T16*>(args.dv) + dv_off(key) : static_cast<T16*>(args.dk) + dk_off(key);
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(lane_base + col + c0, v);
                tmem_ld_wait(v);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack2<BF16>(__uint_as_float(v[2 * i]) * mul, __uint_as_float(v[2 * i + 1]) * mul);
                if (key_in) {
                    uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
                    for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// Element strides (batch, token, head; d contiguous) of a 16-bit [B, N, H, d] tensor.
struct Strides3 {
    long long b, s, h;
};

// D[b,h,q] = sum_c dO[b,q,h,c] O[b,q,h,c] in fp32, and dQ_acc[b,q,h,:] = 0.
// A group of D/8 lanes handles one (b, q, h) row, 8 elements per lane; o and dout
// are addressed through their strides.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_preprocess(const uint16_t* o, const uint16_t* dout, float* Dvec,
                                                          float* dq_acc, size_t acc_f4, int B, int Nq, int Hq,
                                                          bool bf16, Strides3 so, Strides3 sdo) {
    constexpr int kLanes = D / 8;
    const size_t rows = static_cast<size_t>(B) * Nq * Hq;
    const size_t row = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) / kLanes;
    const int sub = threadIdx.x % kLanes;
    float acc = 0.f;
    if (row < rows) {
        const long long rh = static_cast<long long>(row % Hq), rbq = static_cast<long long>(row / Hq);
        const long long rq = rbq % Nq, rb = rbq / Nq;
        const uint4 a = reinterpret_cast<const uint4*>(o + rb * so.b + rq * so.s + rh * so.h)[sub];
        const uint4 c = reinterpret_cast<const uint4*>(dout + rb * sdo.b + rq * sdo.s + rh * sdo.h)[sub];
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float a0, a1, c0, c1;
            if (bf16) {
                a0 = __uint_as_float(av[i] << 16);
                a1 = __uint_as_float(av[i] & 0xFFFF0000u);
                c0 = __uint_as_float(cv[i] << 16);
                c1 = __uint_as_float(cv[i] & 0xFFFF0000u);
            } else {
                a0 = __half2float(__ushort_as_half(static_cast<unsigned short>(av[i] & 0xFFFFu)));
                a1 = __half2float(__ushort_as_half(static_cast<unsigned short>(av[i] >> 16)));
                c0 = __half2float(__ushort_as_half(static_cast<unsigned short>(cv[i] & 0xFFFFu)));
                c1 = __half2float(__ushort_as_half(static_cast<unsigned short>(cv[i] >> 16)));
            }
            acc = fmaf(a0, c0, acc);
            acc = fmaf(a1, c1, acc);
        }
    }
    // Zero the dQ accumulator (acc_f4 float4s; its layout depends on d).
    {
        const size_t nthreads = static_cast<size_t>(gridDim.x) * blockDim.x;
        float4* z = reinterpret_cast<float4*>(dq_acc);
        for (size_t g = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < acc_f4; g += nthreads)
            z[g] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (row < rows && sub == 0) {
        // row = (b * Nq + q) * Hq + h  ->  D layout [B, Hq, Nq]
        const size_t h = row % Hq;
        const size_t bq = row / Hq;
        const size_t q = bq % Nq;
        const size_t bb = bq / Nq;
        Dvec[(bb * Hq + h) * Nq + q] = acc;
    }
}

// dq = dtype(scale * dq_acc) for d = 64 (accumulator [B, Nq, Hq, 64]), 8 elements
// per thread, dq addressed through its strides.
__global__ void __launch_bounds__(256) fa_bwd_dq_convert(const float* dq_acc, uint16_t* dq, size_t n8, float scale,
                                                          bool bf16, int Nq, int Hq, Strides3 sdq,
                                                          const int* cu_q = nullptr) {
    const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n8) return;
    const size_t row = i / 8;  // (b Nq + q) Hq + h; 8 threads per 64-value row
    const long long h = static_cast<long long>(row % Hq), bq = static_cast<long long>(row / Hq);
    const long long b = bq / Nq, q = bq % Nq;
    uint16_t* dst;
    if (cu_q) {  // varlen: Nq = max_seqlen_q; rows past the sequence's length are padding
        if (q >= cu_q[b + 1] - cu_q[b]) return;
        dst = dq + (cu_q[b] + q) * sdq.s + h * sdq.h + (i % 8) * 8;
    } else {
        dst = dq + b * sdq.b + q * sdq.s + h * sdq.h + (i % 8) * 8;
    }
    const float4 a = reinterpret_cast<const float4*>(dq_acc)[2 * i];
    const float4 c = reinterpret_cast<const float4*>(dq_acc)[2 * i + 1];
    uint4 out;
    if (bf16) {
        out = make_uint4(pack2<true>(a.x * scale, a.y * scale), pack2<true>(a.z * scale, a.w * scale),
                         pack2<true>(c.x * scale, c.y * scale), pack2<true>(c.z * scale, c.w * scale));
    } else {
        out = make_uint4(pack2<false>(a.x * scale, a.y * scale), pack2<false>(a.z * scale, a.w * scale),
                         pack2<false>(c.x * scale, c.y * scale), pack2<false>(c.z * scale, c.w * scale));
    }
    *reinterpret_cast<uint4*>(dst) = out;
}

// The d = 128 accumulator keeps four consecutive queries of one head-dimension
// index together: element (b, h, q, c) sits at ((b Hq + h) nq4 + q / 4) 512 +
// 4 c + q % 4, so a warp of the backward main kernel (lane = c) adds four
// queries with one coalesced 512-byte vector reduction. One thread here turns
// head-dimension indices 2p, 2p + 1 of a group of four queries into dQ[token, h, :]:
// token q of batch b for fixed length, packed row cu_q[b] + q for varlen (cu_q
// non-null; b is the sequence, Nq the max_seqlen bound), addressed through dq's
// strides (varlen: the token stride only).
__global__ void __launch_bounds__(256) fa_bwd_dq_convert_g4(const float* dq_acc, uint16_t* dq, const int* cu_q,
                                                             int B, int Hq, int Nq, int nq4, float scale, bool bf16,
                                                             Strides3 sdq) {
    const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // (b, h, g, p)
    const size_t groups = static_cast<size_t>(B) * Hq * nq4;
    if (i >= groups * 64) return;
    const int p = static_cast<int>(i & 63);
    const size_t bhg = i >> 6;
    const int g = static_cast<int>(bhg % nq4);
    const size_t bh = bhg / nq4;
    const int h = static_cast<int>(bh % Hq);
    const int b = static_cast<int>(bh / Hq);
    int q_len = Nq;
    long long base = b * sdq.b;  // token 0 of this batch / sequence
    if (cu_q) {
        base = static_cast<long long>(cu_q[b]) * sdq.s;
        q_len = min(cu_q[b + 1] - cu_q[b], Nq);
    }
    const float4* src = reinterpret_cast<const float4*>(dq_acc) + bhg * 128 + 2 * p;
    const float4 a = src[0], c = src[1];
    const float lo[4] = {a.x, a.y, a.z, a.w}, hi[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int q = 4 * g + j;
        if (q >= q_len) break;
        const uint32_t v = bf16 ? pack2<true>(lo[j] * scale, hi[j] * scale) : pack2<false>(lo[j] * scale, hi[j] * scale);
        reinterpret_cast<uint32_t*>(dq + base + q * sdq.s + h * sdq.h)[p] = v;
    }
}

}  // namespace fa
