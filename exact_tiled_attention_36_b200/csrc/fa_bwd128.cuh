// fa_bwd128.cuh: backward main kernel for d = 128 (same mathematics as
// fa_bwd_kernel in fa_bwd.cuh).
//
// One CTA owns a 128-key tile K_j, V_j of one KV head and walks every 128-row
// query tile Q_i, dO_i of the group's query heads. Per query tile:
//     S^T  = K_j Q_i^T,  dP^T = V_j dO_i^T               (TMEM, 128 x 128 fp32 each)
//     P^T  = 2^(S^T c - L log2 e),  dS^T = P^T o (dP^T - D)
//     dV += P^T dO_i,  dK += dS^T Q_i                      (TMEM accumulators)
//     dQ_i^T = K_j^T dS^T                                 (TMEM, 128 (d) x 128 fp32)
// Every tensor-core product has N = 128 (a 64-wide N runs the tensor core at
// two thirds of its rate or less), so only one query tile is in flight in
// TMEM; the overlap comes from the order of the products instead: the MMA
// thread issues S^T of tile i + 1 right behind dV of tile i, so the softmax of
// tile i + 1 runs while dK and dQ^T of tile i are on the tensor core.
//
// Warp roles (512 threads): warp 0 TMA producer, warp 1 TMEM allocation and the
// single MMA-issuing thread, warps 2-3 idle; warps 4-7 and 8-11 the compute
// warpgroups (warpgroup w owns query columns [64 w, 64 w + 64) of S^T / dP^T,
// and writes dV (w = 0) or dK (w = 1) at the end); warps 12-15 the dQ
// warpgroup, which moves dQ_i^T from TMEM to registers, releases its columns,
// then adds it into the fp32 accumulator with vector reductions.
//
// TMEM columns (512): [0,128) S^T, later P^T as 16-bit pairs in [0,32) and
// [64,96); [128,256) dP^T, later dS^T pairs in [128,160) and [192,224), later
// dQ^T; [256,384) dV; [384,512) dK.
#pragma once

#include "fa_bwd.cuh"

namespace fa {

constexpr int kBwd128Threads = 512;
constexpr int kBwd128RegsOther = 96;     // warps 0-3
constexpr int kBwd128RegsCompute = 136;  // warps 4-11
constexpr int kBwd128RegsDrain = 144;    // warps 12-15
// setmaxnreg.inc waits until the registers it asks for are free, so the launch
// must hold at least the sum of the split (the host checks this).
constexpr int kBwd128MinLaunchRegs =
    (128 * kBwd128RegsOther + 256 * kBwd128RegsCompute + 128 * kBwd128RegsDrain + kBwd128Threads - 1) /
    kBwd128Threads;

struct Bwd128Cfg {
    static constexpr int D = 128;
    static constexpr int kSlabBytes = 128 * 128;
    static constexpr int kTileBytes = 2 * kSlabBytes;     // 128 rows x 128, 16-bit
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kKOff + kTileBytes;
    static constexpr int kQOff = kVOff + kTileBytes;       // 2 stages
    static constexpr int kDOOff = kQOff + 2 * kTileBytes;  // 2 stages
    static constexpr int kDSOff = kDOOff + 2 * kTileBytes;  // dS^T [128 keys x 128 q], two 64-query slabs
    static constexpr int kLDOff = kDSOff + 2 * kSlabBytes;  // [warpgroup][stage][L 64 | D 64] fp32
    static constexpr int kBarOff = kLDOff + 2048;
    static constexpr int kNumBars = 18;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// TMEM column of the 16-bit pairs of query chunk kk (16 queries) of P^T or
// dS^T: warpgroup w wrote queries [64 w, 64 w + 64) as 32 pair columns at
// region + 64 w.
__device__ __forceinline__ uint32_t pair_col(int kk) {
    return static_cast<uint32_t>(kk < 4 ? kk * 8 : 64 + (kk - 4) * 8);
}

template <bool BF16, bool CAUSAL, bool VARLEN>
__global__ void __launch_bounds__(kBwd128Threads, 1)
    fa_bwd128_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const BwdArgs args) {
    using C = Bwd128Cfg;
    constexpr int D = C::D;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (!smem_base_ok(smem, args.err)) return;

    // Grid order. Without the causal mask, and under it when each KV head serves one
    // query head (args.kt_fast), the grid is (key tiles, Hkv, sequences): the key tiles of a
    // (sequence, KV head) run together, key tile kt at query tile kt + t at time t, so
    // their dQ reductions land on neighbouring lines that stay in the L2. Under the causal
    // mask with larger groups the walks are longer (group x query tiles), and the grid is
    // (Hkv, sequences, key tiles): the first key tiles of every pair, the longest walks,
    // are dispatched first, so no long walk starts near the end.
    const bool kt_x = !CAUSAL || args.kt_fast;
    const int kt = kt_x ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.z);
    const int hk = kt_x ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.x);
    const int b = kt_x ? static_cast<int>(blockIdx.z) : static_cast<int>(blockIdx.y);
    const int k0 = kt * 128;
    // Rows of this sequence: fixed length, or varlen (b is the sequence; its rows
    // start at q_row0 / k_row0 of the packed buffers).
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
    int i0, n_i;  // the query tiles that see some key of this tile
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

    // Query tile of iteration it (query head hk * group + it / n_i). Without the
    // causal mask the key tiles of a KV head start their walk at different query
    // tiles, so concurrent CTAs add into different rows of the dQ accumulator.
    const int rot = CAUSAL ? 0 : kt % n_i;
    auto qtile = [&](int it_) {
        const int x = it_ % n_i + rot;
        return i0 + (x >= n_i ? x - n_i : x);
    };

    uint8_t* sK = smem + C::kKOff;
    uint8_t* sV = smem + C::kVOff;
    uint8_t* sQ = smem + C::kQOff;
    uint8_t* sDO = smem + C::kDOOff;
    uint8_t* sDS = smem + C::kDSOff;
    float* sLD = reinterpret_cast<float*>(smem + C::kLDOff);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* kv_full = bars;
    uint64_t* q_full = bars + 1;   // [2 stages]
    uint64_t* q_empty = bars + 3;  // [2 stages]
    uint64_t* s_full = bars + 5;
    uint64_t* dp_full = bars + 6;
    uint64_t* p_ready = bars + 7;
    uint64_t* ds_ready = bars + 8;
    uint64_t* dq_full = bars + 9;
    uint64_t* dq_free = bars + 10;
    uint64_t* ld_full = bars + 11;  // [warpgroup * 2 + stage]
    uint64_t* fin = bars + 15;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    int* abort_flag = reinterpret_cast<int*>(smem + C::kMiscOff + 4);

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(p_ready, 256);
        mbar_init(ds_ready, 256);
        mbar_init(dq_full, 1);
        mbar_init(dq_free, 128);
        for (int i = 0; i < 4; ++i) mbar_init(&ld_full[i], 64);
        mbar_init(fin, 1);
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

    if (warp < 4) {
        setmaxnreg_dec<kBwd128RegsOther>();
        if (warp == 0 && lane == 0) {
            // -------------------------------------------------------- producer
            mbar_arrive_expect_tx(kv_full, 2 * C::kTileBytes);
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                tma_load_4d(sK + s * C::kSlabBytes, &tm_k, kv_full, s * 64, hk, k_row0 + k0, tma_b);
                tma_load_4d(sV + s * C::kSlabBytes, &tm_v, kv_full, s * 64, hk, k_row0 + k0, tma_b);
            }
            int issued = 0;
            for (int it = 0; it < n_it; ++it) {
                const int st = it & 1;
                const int h = hk * args.group + it / n_i;
                const int q0 = qtile(it) * 128;
                if (!mbar_wait(&q_empty[st], ((it >> 1) & 1) ^ 1u, wc, 61)) break;
                mbar_arrive_expect_tx(&q_full[st], 2 * C::kTileBytes);
#pragma unroll
                for (int s = 0; s < 2; ++s) {
                    tma_load_4d(sQ + st * C::kTileBytes + s * C::kSlabBytes, &tm_q, &q_full[st], s * 64, h,
                                q_row0 + q0, tma_b);
                    tma_load_4d(sDO + st * C::kTileBytes + s * C::kSlabBytes, &tm_do, &q_full[st], s * 64, h,
                                q_row0 + q0, tma_b);
                }
                ++issued;
                // Warm the L2 with the tiles two iterations ahead.
                if (it + 2 < n_it) {
                    const int h2 = hk * args.group + (it + 2) / n_i;
                    const int q2 = qtile(it + 2) * 128;
#pragma unroll
                    for (int s = 0; s < 2; ++s) {
                        tma_prefetch_l2_4d(&tm_q, s * 64, h2, q_row0 + q2, tma_b);
                        tma_prefetch_l2_4d(&tm_do, s * 64, h2, q_row0 + q2, tma_b);
                    }
                }
            }
            mbar_wait_drain(kv_full, 0);
            for (int st = 0; st < 2; ++st)
                if (issued > st) mbar_wait_drain(&q_full[st], (((issued - 1 - st) / 2 * 2 + st) >> 1) & 1);
        }
        if (warp == 1 && lane == 0) {
            // ------------------------------------------------------ MMA issuer
            constexpr uint32_t id_ss = idesc_f16(128, 128, BF16, false, false);  // S^T, dP^T: keys x queries
            constexpr uint32_t id_tm = idesc_f16(128, D, BF16, false, true);     // dV, dK: A from TMEM
            constexpr uint32_t id_dq = idesc_f16(128, 128, BF16, true, true);    // dQ^T: A = K^T, B = dS^T
            const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV), ds_addr = smem_u32(sDS);
            // S^T = K Q^T or dP^T = V dO^T: 8 products over d.
            auto issue_sd = [&](uint32_t col, uint32_t a_addr, uint32_t b_addr) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kSlabBytes + (kk & 3) * 32;
                    mma_ss(tmem + col, sdesc_sw128(a_addr + off, 16, 1024), sdesc_sw128(b_addr + off, 16, 1024),
                           id_ss, kk > 0 ? 1u : 0u);
                }
            };
            bool ok = mbar_wait(kv_full, 0, wc, 62) && mbar_wait(&q_full[0], 0, wc, 63);
            if (ok) {
                tc_fence_after();
                issue_sd(C::kColS, k_addr, smem_u32(sQ));
                tc_commit(s_full);
            }
            for (int it = 0; ok && it < n_it; ++it) {
                const int st = it & 1;
                const uint32_t q_addr = smem_u32(sQ + st * C::kTileBytes);
                const uint32_t do_addr = smem_u32(sDO + st * C::kTileBytes);
                // dP^T_it: its columns held dQ^T of the previous tile until the dQ
                // warpgroup took it into registers.
                if (it > 0 && !(ok = mbar_wait(dq_free, (it - 1) & 1, wc, 64))) break;
                tc_fence_after();
                issue_sd(C::kColDP, v_addr, do_addr);
                tc_commit(dp_full);
                // dV += P^T dO once the compute warpgroups have written P^T.
                if (!(ok = mbar_wait(p_ready, it & 1, wc, 65))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + C::kColDV, tmem + C::kColS + pair_col(kk),
                           sdesc_sw128(do_addr + kk * 2048, C::kSlabBytes, 1024), id_tm, (it > 0 || kk > 0) ? 1u : 0u);
                // S^T of the next tile right behind dV (it overwrites P^T after dV has
                // read it: one thread's tcgen05.mma operations execute in issue order),
                // unless its Q tile has not arrived yet; then it follows dQ^T.
                const bool has_next = it + 1 < n_it;
                const int nst = (it + 1) & 1;
                bool s_next = false;
                if (has_next && mbar_try_wait(smem_u32(&q_full[nst]), ((it + 1) >> 1) & 1)) {
                    tc_fence_after();
                    issue_sd(C::kColS, k_addr, smem_u32(sQ + nst * C::kTileBytes));
                    tc_commit(s_full);
                    s_next = true;
                }
                if (!(ok = mbar_wait(ds_ready, it & 1, wc, 66))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + C::kColDK, tmem + C::kColDP + pair_col(kk),
                           sdesc_sw128(q_addr + kk * 2048, C::kSlabBytes, 1024), id_tm, (it > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&q_empty[st]);  // dQ^T reads neither Q nor dO
                // dQ^T = K^T dS^T over the dP^T columns (dK has read dS^T: issue order).
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tmem + C::kColDP, sdesc_sw128(k_addr + kk * 2048, C::kSlabBytes, 1024),
                           sdesc_sw128(ds_addr + kk * 2048, C::kSlabBytes, 1024), id_dq, kk > 0 ? 1u : 0u);
                tc_commit(dq_full);
                if (has_next && !s_next) {
                    if (!(ok = mbar_wait(&q_full[nst], ((it + 1) >> 1) & 1, wc, 67))) break;
                    tc_fence_after();
                    issue_sd(C::kColS, k_addr, smem_u32(sQ + nst * C::kTileBytes));
                    tc_commit(s_full);
                }
            }
            tc_commit(fin);
            mbar_wait_drain(fin, 0);
        }
    } else if (warp < 12) {
        // ------------------------------------------------------------ compute warpgroups
        setmaxnreg_inc<kBwd128RegsCompute>();
        const int w = (warp - 4) >> 2;  // query columns [64 w, 64 w + 64)
        const int w4 = warp & 3;
        const int r = w4 * 32 + lane;  // TMEM lane: key row
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(w4 * 32) << 16);
        const int key = k0 + r;
        const bool key_in = key < Nk;                          // a row of dK / dV to write
        const bool key_ok = key_in && key_kept(args, b, key);  // a key that takes part
        const bool keys_masked = tile_keys_masked(args, b, k0, Nk);  // uniform
        int qlim, qlim_hi;  // queries [qlim, qlim_hi) see this key
        query_range<CAUSAL>(args, key, Nq, Nk, qlim, qlim_hi);
        // Every key of the tile sees queries [qall_lo, qall_hi): slices inside need no mask.
        // qlo grows with the key, so the last key's is the largest; qhi grows too except
        // that anchor keys see every later query, so the smallest is that of the tile's
        // first key that is not an anchor (its first key if none is).
        int qall_lo, qdummy, qdummy2, qall_hi;
        const int k_last = min(k0 + 127, Nk - 1);
        query_range<CAUSAL>(args, k_last, Nq, Nk, qall_lo, qdummy);
        query_range<CAUSAL>(args, min(max(k0, args.n_anchor), k_last), Nq, Nk, qdummy2, qall_hi);
        const float sl2 = args.scale_log2;
        constexpr float kLog2eF = 1.4426950408889634074f;
        // -L log2 e and -D of query 64 w + r of iteration it_, loaded one iteration
        // ahead so the global-load latency overlaps the previous tile's work.
        auto load_ld = [&](int it_, float& l2, float& dd) {
            l2 = -INFINITY;
            dd = 0.f;
            if (r < 64 && it_ < n_it) {
                const int q = qtile(it_) * 128 + w * 64 + r;
                if (q < Nq) {
                    const int hq = hk * args.group + it_ / n_i;
                    const size_t row = VARLEN ? static_cast<size_t>(hq) * args.total_q + q_row0 + q
                                              : (static_cast<size_t>(b) * args.Hq + hq) * Nq + q;
                    const float L = __ldg(args.lse + row);
                    l2 = (L == -INFINITY) ? -INFINITY : -L * kLog2eF;  // a row that saw no key has P = 0
                    dd = -__ldg(args.D + row);
                }
            }
        };
        float next_l2, next_dd;
        load_ld(0, next_l2, next_dd);
        uint8_t* ds_rows = sDS + w * C::kSlabBytes + (r >> 3) * 1024 + (r & 7) * 128;
        const uint64_t c2 = f2_pack(sl2, sl2);
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const int qs = qtile(it) * 128 + w * 64;  // first query of this warpgroup's columns
            // Buffer (w, it & 1) is rewritten at it + 2, after every thread of the
            // warpgroup has passed dp_full of it + 1, which the MMA thread commits only
            // after ds_ready of it.
            float* sL = sLD + (w * 2 + (it & 1)) * 128;
            float* sD = sL + 64;
            if (r < 64) {
                sL[r] = next_l2;
                sD[r] = next_dd;
                mbar_arrive(&ld_full[w * 2 + (it & 1)]);
            }
            load_ld(it + 1, next_l2, next_dd);
            ok = warp_all(mbar_wait(&ld_full[w * 2 + (it & 1)], (it >> 1) & 1, wc, 68));
            if (!ok) break;
            ok = warp_all(mbar_wait(s_full, it & 1, wc, 69));
            if (!ok) break;
            tc_fence_after();
            // Masks matter only on the tile holding key Nk - 1 and, under a window mask
            // (causal included), on query columns outside some key's window (uniform per
            // warpgroup).
            const bool need_mask =
                (k0 + 128 > Nk) || keys_masked || (CAUSAL && (qs < qall_lo || qs + 64 > qall_hi));
            float pf[64];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t sv[32];
                tmem_ld32(lane_base + C::kColS + w * 64 + cc * 32, sv);
                tmem_ld_wait(sv);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const ulonglong2 nl = *reinterpret_cast<const ulonglong2*>(sL + cc * 32 + e);
                    float p[4];
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const int u = e + 2 * h2;
                        const uint64_t y = f2_fma(f2_pack(__uint_as_float(sv[u]), __uint_as_float(sv[u + 1])), c2,
                                                  h2 ? nl.y : nl.x);
                        float y0, y1;
                        f2_unpack(y, y0, y1);
                        p[2 * h2] = ex2_approx(y0);
                        p[2 * h2 + 1] = ex2_approx(y1);
                    }
                    if (need_mask) {
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            bool vis = key_ok;
                            if (CAUSAL) {
                                const int qv = qs + cc * 32 + e + u;
                                vis = vis && qv >= qlim && qv < qlim_hi;
                            }
                            p[u] = vis ? p[u] : 0.f;
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) pf[cc * 32 + e + u] = p[u];
                    pk[e >> 1] = pack2<BF16>(p[0], p[1]);
                    pk[(e >> 1) + 1] = pack2<BF16>(p[2], p[3]);
                }
                // 16-bit pairs over columns this thread has already read (query
                // 32 cc + e lands in column 16 cc + e / 2 of the warpgroup's region).
                tmem_st16(lane_base + C::kColS + w * 64 + cc * 16, pk);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(p_ready);
            ok = warp_all(mbar_wait(dp_full, it & 1, wc, 70));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t pv[32];
                tmem_ld32(lane_base + C::kColDP + w * 64 + cc * 32, pv);
                tmem_ld_wait(pv);
                uint32_t dk16[16];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const ulonglong2 nd = *reinterpret_cast<const ulonglong2*>(sD + cc * 32 + e);
                    float ds[4];
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const int u = e + 2 * h2;
                        const uint64_t dpm = f2_add(f2_pack(__uint_as_float(pv[u]), __uint_as_float(pv[u + 1])),
                                                    h2 ? nd.y : nd.x);
                        f2_unpack(f2_mul(f2_pack(pf[cc * 32 + u], pf[cc * 32 + u + 1]), dpm), ds[2 * h2],
                                  ds[2 * h2 + 1]);
                    }
                    dk16[e >> 1] = pack2<BF16>(ds[0], ds[1]);
                    dk16[(e >> 1) + 1] = pack2<BF16>(ds[2], ds[3]);
                }
                tmem_st16(lane_base + C::kColDP + w * 64 + cc * 16, dk16);
                // dS^T row of this key into the MN-major operand of dQ^T: 128 B per key
                // (64 queries), 16-byte chunks swizzled by key % 8.
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int chunk = (cc * 4 + u) ^ (r & 7);
                    *reinterpret_cast<uint4*>(ds_rows + chunk * 16) =
                        make_uint4(dk16[4 * u], dk16[4 * u + 1], dk16[4 * u + 2], dk16[4 * u + 3]);
                }
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(ds_ready);
        }
        if (ok) ok = warp_all(mbar_wait(fin, 0, wc, 71));
        if (ok) {
            tc_fence_after();
            // Warpgroup 0 writes dV, warpgroup 1 writes dK = scale * (dS^T Q).
            const uint32_t col = w == 0 ? C::kColDV : C::kColDK;
            const float mul = w == 0 ? 1.f : args.scale;
            T16* dst = w == 0 ? static_cast<T16*>(args.dv) + dv_off(key) : static_cast<T16*>(args.dk) + dk_off(key);
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
    } else {
        // ------------------------------------------------------------ dQ warpgroup
        setmaxnreg_inc<kBwd128RegsDrain>();
        const int w4 = warp & 3;
        const int r = w4 * 32 + lane;  // TMEM lane: head-dimension index
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(w4 * 32) << 16);
        for (int it = 0; it < n_it; ++it) {
            const int h = hk * args.group + it / n_i;
            const int q0 = qtile(it) * 128;
            if (!warp_all(mbar_wait(dq_full, it & 1, wc, 72))) break;
            tc_fence_after();
            // The whole tile comes into registers first, so the MMA thread can reuse
            // its columns for the next dP^T while the reductions wait on the L2.
            uint32_t v0[32], v1[32], v2[32], v3[32];
            tmem_ld32(lane_base + C::kColDP + 0, v0);
            tmem_ld32(lane_base + C::kColDP + 32, v1);
            tmem_ld32(lane_base + C::kColDP + 64, v2);
            tmem_ld32(lane_base + C::kColDP + 96, v3);
            tmem_ld_wait(v0);
            tmem_ld_wait(v1);
            tmem_ld_wait(v2);
            tmem_ld_wait(v3);
            tc_fence_before();
            mbar_arrive(dq_free);
            // Column c is query q0 + c. Four consecutive queries of index r are adjacent
            // in the accumulator: a warp adds 4 queries x 32 indices with one 512-byte
            // vector reduction.
            float* dst = args.dq_acc + ((static_cast<size_t>(b) * args.Hq + h) * args.nq4 + q0 / 4) * 512 + r * 4;
            const int g_end = (Nq - q0 + 3) / 4;  // groups of four holding a query < Nq
            auto add8 = [&](const uint32_t(&v)[32], int g0) {
#pragma unroll
                for (int g = 0; g < 8; ++g)
                    if (g0 + g < g_end)
                        red_add_v4(dst + (g0 + g) * 512, __uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1]),
                                   __uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3]));
            };
            add8(v0, 0);
            add8(v1, 8);
            add8(v2, 16);
            add8(v3, 24);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace fa
