// fa_bwd_pp.cuh: backward main kernel for d = 128 with two query sub-tiles in
// ping-pong (same mathematics as fa_bwd_kernel in fa_bwd.cuh).
//
// One CTA owns a 128-key tile K_j, V_j of one KV head. Every 128-row query
// tile Q_i, dO_i it visits is split into two 64-row sub-tiles t = 0, 1, each
// owned by one compute warpgroup. Per sub-tile:
//     S^T_t  = K_j Q_t^T,  dP^T_t = V_j dO_t^T          (TMEM, 128 x 64 fp32 each)
//     P^T_t  = 2^(S^T_t c - L log2 e),  dS^T_t = P^T_t o (dP^T_t - D)
//     dV += P^T_t dO_t,  dK += dS^T_t Q_t                 (TMEM accumulators)
//     dQ^T_t = K_j^T dS^T_t                              (TMEM, 128 (d) x 64 fp32)
// While one warpgroup turns its S^T/dP^T into P^T/dS^T, the tensor core runs
// the other sub-tile's products, and while a warpgroup drains its dQ^T into
// the fp32 accumulator (coalesced: lane = head-dimension index, consecutive
// lanes hit consecutive addresses) the other sub-tile's next products run.
//
// TMEM columns (512): [0,64) S^T_0, later P^T_0 (first 32), later dQ^T_0;
// [64,128) the same for sub-tile 1; [128,192) dP^T_0, later dS^T_0;
// [192,256) dP^T_1, later dS^T_1; [256,384) dV; [384,512) dK.
// Each warpgroup only touches its own sub-tile's columns until the epilogue.
#pragma once

#include "fa_bwd.cuh"

namespace fa {

struct BwdPPCfg {
    static constexpr int D = 128;
    static constexpr int kSlabBytes = 128 * 128;
    static constexpr int kTileBytes = 2 * kSlabBytes;     // 128 rows x 128, 16-bit
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kKOff + kTileBytes;
    static constexpr int kQOff = kVOff + kTileBytes;       // 2 stages
    static constexpr int kDOOff = kQOff + 2 * kTileBytes;  // 2 stages
    static constexpr int kDSOff = kDOOff + 2 * kTileBytes;  // 2 sub-tiles x [128 keys x 64 q] 16-bit
    static constexpr int kLDOff = kDSOff + 2 * kSlabBytes;  // [sub-tile][stage][L2 64 | D 64] fp32
    static constexpr int kBarOff = kLDOff + 2048;
    static constexpr int kNumBars = 18;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

__device__ __forceinline__ void red_add_f32(float* addr, float v) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}

template <bool BF16, bool CAUSAL>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_pp_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const BwdArgs args) {
    using C = BwdPPCfg;
    constexpr int D = C::D;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (!smem_base_ok(smem, args.err)) return;

    const int kt = CAUSAL ? static_cast<int>(blockIdx.z) : static_cast<int>(blockIdx.x);
    const int hk = CAUSAL ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.y);
    const int b = CAUSAL ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.z);
    const int k0 = kt * 128;
    const int Nq = args.Nq, Nk = args.Nk;
    const int n_qt = (Nq + 127) / 128;
    int i0 = 0;
    if (CAUSAL) {
        const int qmin = k0 - (Nk - Nq);  // smallest query that sees key k0
        i0 = qmin <= 0 ? 0 : qmin / 128;
    }
    const int n_i = n_qt > i0 ? n_qt - i0 : 0;
    const int n_it = args.group * n_i;

    using T16 = uint16_t;
    const int warp = warp_id();
    const int lane = lane_id();

    if (n_it == 0) {  // no query sees this key tile: dK = dV = 0
        if (threadIdx.x < 128) {
            const int key = k0 + static_cast<int>(threadIdx.x);
            if (key < Nk) {
                const size_t off = ((static_cast<size_t>(b) * Nk + key) * args.Hkv + hk) * D;
                uint4* a = reinterpret_cast<uint4*>(static_cast<T16*>(args.dk) + off);
                uint4* c = reinterpret_cast<uint4*>(static_cast<T16*>(args.dv) + off);
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
    float* sLD = reinterpret_cast<float*>(smem + C::kLDOff);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* kv_full = bars;
    uint64_t* q_full = bars + 1;     // [2 stages]
    uint64_t* q_empty = bars + 3;    // [2 stages]
    uint64_t* s_full = bars + 5;     // [2 sub-tiles]
    uint64_t* ds_ready = bars + 7;   // [2]
    uint64_t* dq_full = bars + 9;    // [2]
    uint64_t* dq_free = bars + 11;   // [2]
    uint64_t* ld_full = bars + 13;   // [sub-tile * 2 + stage]
    uint64_t* fin = bars + 17;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    int* abort_flag = reinterpret_cast<int*>(smem + C::kMiscOff + 4);

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&ds_ready[i], 128);
            mbar_init(&dq_full[i], 1);
            mbar_init(&dq_free[i], 128);
        }
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

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_expect_tx(kv_full, 2 * C::kTileBytes);
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                tma_load_4d(sK + s * C::kSlabBytes, &tm_k, kv_full, s * 64, hk, k0, b);
                tma_load_4d(sV + s * C::kSlabBytes, &tm_v, kv_full, s * 64, hk, k0, b);
            }
            int issued = 0;
            for (int it = 0; it < n_it; ++it) {
                const int st = it & 1;
                const int h = hk * args.group + it / n_i;
                const int q0 = (i0 + it % n_i) * 128;
                if (!mbar_wait(&q_empty[st], ((it >> 1) & 1) ^ 1u, wc, 41)) break;
                mbar_arrive_expect_tx(&q_full[st], 2 * C::kTileBytes);
#pragma unroll
                for (int s = 0; s < 2; ++s) {
                    tma_load_4d(sQ + st * C::kTileBytes + s * C::kSlabBytes, &tm_q, &q_full[st], s * 64, h, q0, b);
                    tma_load_4d(sDO + st * C::kTileBytes + s * C::kSlabBytes, &tm_do, &q_full[st], s * 64, h, q0, b);
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
            constexpr uint32_t id_sd = idesc_f16(128, 64, BF16, false, false);   // S^T, dP^T: 128 keys x 64 q
            constexpr uint32_t id_tm = idesc_f16(128, D, BF16, false, true);     // dV, dK: A from TMEM
            constexpr uint32_t id_dq = idesc_f16(128, 64, BF16, true, true);     // dQ^T: A = K^T, B = dS^T
            const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
            bool ok = mbar_wait(kv_full, 0, wc, 42);
            for (int it = 0; ok && it < n_it; ++it) {
                const int st = it & 1;
                if (!(ok = mbar_wait(&q_full[st], (it >> 1) & 1, wc, 43))) break;
                const uint32_t q_addr = smem_u32(sQ + st * C::kTileBytes);
                const uint32_t do_addr = smem_u32(sDO + st * C::kTileBytes);
                // S^T_t and dP^T_t of both sub-tiles. Sub-tile t's columns are free
                // once its previous dQ^T has been drained.
                for (int t = 0; ok && t < 2; ++t) {
                    if (it > 0 && !(ok = mbar_wait(&dq_free[t], (it - 1) & 1, wc, 44))) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::kSlabBytes + (kk & 3) * 32;
                        mma_ss(tmem + C::kColS + t * 64, sdesc_sw128(k_addr + off, 16, 1024),
                               sdesc_sw128(q_addr + t * 8192 + off, 16, 1024), id_sd, kk > 0 ? 1u : 0u);
                    }
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::kSlabBytes + (kk & 3) * 32;
                        mma_ss(tmem + C::kColDP + t * 64, sdesc_sw128(v_addr + off, 16, 1024),
                               sdesc_sw128(do_addr + t * 8192 + off, 16, 1024), id_sd, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&s_full[t]);
                }
                if (!ok) break;
                // dV, dK from P^T_t / dS^T_t, then dQ^T_t into P^T_t's columns right
                // behind them: tcgen05.mma operations of one thread execute in issue
                // order, so dQ^T_t cannot overwrite P^T_t before dV has read it (the
                // same holds for the next dP^T_t over dS^T_t).
                for (int t = 0; ok && t < 2; ++t) {
                    if (!(ok = mbar_wait(&ds_ready[t], it & 1, wc, 45))) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tmem + C::kColDV, tmem + C::kColS + t * 64 + kk * 8,
                               sdesc_sw128(do_addr + t * 8192 + kk * 2048, C::kSlabBytes, 1024), id_tm,
                               (it > 0 || t > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tmem + C::kColDK, tmem + C::kColDP + t * 64 + kk * 8,
                               sdesc_sw128(q_addr + t * 8192 + kk * 2048, C::kSlabBytes, 1024), id_tm,
                               (it > 0 || t > 0 || kk > 0) ? 1u : 0u);
                    const uint32_t ds_addr = smem_u32(sDS + t * C::kSlabBytes);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + C::kColS + t * 64, sdesc_sw128(k_addr + kk * 2048, C::kSlabBytes, 1024),
                               sdesc_sw128(ds_addr + kk * 2048, C::kSlabBytes, 1024), id_dq, kk > 0 ? 1u : 0u);
                    tc_commit(&dq_full[t]);
                }
                tc_commit(&q_empty[st]);
            }
            tc_commit(fin);
            mbar_wait_drain(fin, 0);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ compute warpgroups
        const int t = (warp - 4) >> 2;  // sub-tile owned by this warpgroup
        const int w4 = warp & 3;
        const int r = w4 * 32 + lane;  // TMEM lane: key row (S^T, dP^T, dV, dK) or head-dim index (dQ^T)
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(w4 * 32) << 16);
        const int key = k0 + r;
        const bool key_ok = key < Nk;
        const int qlim = key - (Nk - Nq);  // smallest query that sees this key
        const float sl2 = args.scale_log2;
        constexpr float kLog2eF = 1.4426950408889634074f;
        // L (log2 units) and D of query qs + r, loaded one iteration ahead so the
        // global-load latency overlaps the previous sub-tile's work.
        // Stored negated: -L log2 e (so P = 2^(S c + that) is one FMA and an exp) and -D.
        auto load_ld = [&](int it_, float& l2, float& dd) {
            l2 = -INFINITY;
            dd = 0.f;
            if (r < 64 && it_ < n_it) {
                const int q = (i0 + it_ % n_i) * 128 + t * 64 + r;
                if (q < Nq) {
                    const size_t row = (static_cast<size_t>(b) * args.Hq + hk * args.group + it_ / n_i) * Nq + q;
                    const float L = __ldg(args.lse + row);
                    l2 = (L == -INFINITY) ? -INFINITY : -L * kLog2eF;  // a row that saw no key has P = 0
                    dd = -__ldg(args.D + row);
                }
            }
        };
        float next_l2, next_dd;
        load_ld(0, next_l2, next_dd);
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const int h = hk * args.group + it / n_i;
            const int qs = (i0 + it % n_i) * 128 + t * 64;  // first query of this sub-tile
            // Buffer (t, it & 1) is rewritten at it + 2, when every thread of this
            // warpgroup has arrived on ds_ready for it + 1.
            float* sL = sLD + (t * 2 + (it & 1)) * 128;
            float* sD = sL + 64;
            if (r < 64) {
                sL[r] = next_l2;
                sD[r] = next_dd;
                mbar_arrive(&ld_full[t * 2 + (it & 1)]);
            }
            load_ld(it + 1, next_l2, next_dd);
            ok = warp_all(mbar_wait(&ld_full[t * 2 + (it & 1)], (it >> 1) & 1, wc, 47));
            if (!ok) break;
            ok = warp_all(mbar_wait(&s_full[t], it & 1, wc, 48));
            if (!ok) break;
            tc_fence_after();
            uint8_t* ds_rows = sDS + t * C::kSlabBytes + (r >> 3) * 1024 + (r & 7) * 128;
            // Masks matter only on the tile holding key Nk - 1 and, under the causal
            // mask, on sub-tiles that reach below the diagonal (uniform per sub-tile).
            const bool need_mask = (k0 + 128 > Nk) || (CAUSAL && qs < k0 + 127 - (Nk - Nq));
            const uint64_t c2 = f2_pack(sl2, sl2);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t sv[32], pv[32];
                tmem_ld32(lane_base + C::kColS + t * 64 + cc * 32, sv);
                tmem_ld32(lane_base + C::kColDP + t * 64 + cc * 32, pv);
                tmem_ld_wait(sv);
                tmem_ld_wait(pv);
                uint32_t pk[16], dk16[16];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    // pairs of queries through the packed f32x2 FMA, add and multiply
                    const ulonglong2 nl = *reinterpret_cast<const ulonglong2*>(sL + cc * 32 + e);
                    const ulonglong2 nd = *reinterpret_cast<const ulonglong2*>(sD + cc * 32 + e);
                    float p[4], ds[4];
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
                            if (CAUSAL) vis = vis && (qs + cc * 32 + e + u >= qlim);
                            p[u] = vis ? p[u] : 0.f;
                        }
                    }
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const int u = e + 2 * h2;
                        const uint64_t dpm = f2_add(f2_pack(__uint_as_float(pv[u]), __uint_as_float(pv[u + 1])),
                                                    h2 ? nd.y : nd.x);
                        f2_unpack(f2_mul(f2_pack(p[2 * h2], p[2 * h2 + 1]), dpm), ds[2 * h2], ds[2 * h2 + 1]);
                    }
                    pk[e >> 1] = pack2<BF16>(p[0], p[1]);
                    pk[(e >> 1) + 1] = pack2<BF16>(p[2], p[3]);
                    dk16[e >> 1] = pack2<BF16>(ds[0], ds[1]);
                    dk16[(e >> 1) + 1] = pack2<BF16>(ds[2], ds[3]);
                }
                // 16-bit pairs over columns this thread has already read (query 32 cc + e
                // lands in column 16 cc + e / 2 of the sub-tile's region).
                tmem_st16(lane_base + C::kColS + t * 64 + cc * 16, pk);
                tmem_st16(lane_base + C::kColDP + t * 64 + cc * 16, dk16);
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
            mbar_arrive(&ds_ready[t]);
            // Drain dQ^T_t: lane r is head-dimension index r, column c is query qs + c.
            ok = warp_all(mbar_wait(&dq_full[t], it & 1, wc, 49));
            if (!ok) break;
            tc_fence_after();
            const size_t qstride = static_cast<size_t>(args.Hq) * D;
            float* dst = args.dq_acc + (static_cast<size_t>(b) * Nq * args.Hq + h) * D + r +
                         static_cast<size_t>(qs) * qstride;
            const int q_end = Nq - qs;  // queries qs + c with c >= q_end do not exist
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t v[32];
                tmem_ld32(lane_base + C::kColS + t * 64 + cc * 32, v);
                tmem_ld_wait(v);
                if (q_end >= 64) {
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        red_add_f32(dst, __uint_as_float(v[c]));
                        dst += qstride;
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        if (cc * 32 + c < q_end) red_add_f32(dst, __uint_as_float(v[c]));
                        dst += qstride;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&dq_free[t]);
        }
        if (ok) ok = warp_all(mbar_wait(fin, 0, wc, 50));
        if (ok) {
            tc_fence_after();
            // Warpgroup 0 writes dV, warpgroup 1 writes dK = scale * (dS^T Q).
            const uint32_t col = t == 0 ? C::kColDV : C::kColDK;
            const float mul = t == 0 ? 1.f : args.scale;
            T16* dst = static_cast<T16*>(t == 0 ? args.dv : args.dk) +
                       ((static_cast<size_t>(b) * Nk + key) * args.Hkv + hk) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(lane_base + col + c0, v);
                tmem_ld_wait(v);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack2<BF16>(__uint_as_float(v[2 * i]) * mul, __uint_as_float(v[2 * i + 1]) * mul);
                if (key_ok) {
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

}  // namespace fa
