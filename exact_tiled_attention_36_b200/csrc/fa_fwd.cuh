// fa_fwd.cuh: tiled exact attention forward for sm_100a.
//
// One CTA computes one 128-row query tile Q_i of one (batch, query head) and
// walks the key/value tiles K_j, V_j of 128 rows with the online softmax
// ("FlashAttention/zh", section "FlashAttention algorithm"): S_ij = Q_i K_j^T,
// the running row max m and normaliser l, the rescale of the partial output by
// exp(m_old - m_new), the final O_i / l_i and L_i = m_i + log l_i. The loop
// order is query tile outside, key tile inside (the FlashAttention-2 work
// split on the same page, section "variants").
//
// Warp roles (256 threads):
//   warp 0      TMA producer: Q once, then K_j and V_j into NS-deep rings.
//   warp 1      allocates TMEM and issues every tcgen05.mma from one thread:
//               S_j = Q K_j^T into one of two TMEM score buffers (so S_{j+1}
//               is computed while the softmax works on S_j), and
//               O += P_j V_j with P_j read from TMEM; S_{j+2} is issued once
//               P_j V_j has completed, since it reuses P_j's columns.
//   warps 4-7   softmax: thread t owns query row t = TMEM lane t. It loads its
//               row of S_j, masks, takes the row max, forms
//               P = 2^(S * scale * log2 e - m) with the scale folded into one
//               FFMA, writes P as 16-bit pairs over the first half of the same
//               TMEM columns, keeps l (for L) and the sum of the rounded P
//               (which normalises O), rescales its O row in TMEM when m has
//               grown by more than 2^8 since the last rescale (exact: O and l
//               share the stale reference max), and finally writes O / l and L.
//   warps 2-3   idle.
//
// TMEM columns: [0,128) S buffer 0, [128,256) S buffer 1, [256,256+d) O.
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
    float scale_log2;  // scale * log2(e)
    int* err;
};

template <int D>
struct FwdCfg {
    static constexpr int kSlabs = D / 64;        // 64-column slabs of 128 rows x 128 B
    static constexpr int kSlabBytes = 128 * 128;
    static constexpr int kTileBytes = kSlabs * kSlabBytes;
    static constexpr int kStages = (D == 128) ? 3 : 4;
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + kTileBytes;
    static constexpr int kVOff = kKOff + kStages * kTileBytes;
    static constexpr int kBarOff = kVOff + kStages * kTileBytes;
    static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 1 + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16;  // + slack for 1024-B alignment
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O once m grew by > 2^8
constexpr float kLn2 = 0.69314718055994530942f;

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

// Time-bounded wait used only while draining at exit (ignores the abort flag).
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(a, parity)) {
        if (globaltimer_ns() - t0 > 200000000ull) break;
    }
}

template <int D, bool BF16, bool CAUSAL, bool VARLEN>
__global__ void __launch_bounds__(256, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdArgs args) {
    using C = FwdCfg<D>;
    constexpr int S = C::kStages;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (!smem_base_ok(smem, args.err)) return;  // the 128-byte swizzle needs 1024-byte aligned tiles

    // Non-causal grid (q tiles, Hq, batches): neighbouring CTAs share K/V in L2.
    // Causal grid (Hq, batches, q tiles), the last query tile first: CTAs are
    // dispatched heaviest first (longest-processing-time order), so the long
    // tiles do not start in the last wave.
    const int h = CAUSAL ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.y);
    const int bidx = CAUSAL ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.z);
    const int q_tile = CAUSAL ? static_cast<int>(gridDim.z - 1 - blockIdx.z) : static_cast<int>(blockIdx.x);
    const int q0 = q_tile * 128;

    int q_len, k_len, q_row0, k_row0, tma_b;
    if constexpr (VARLEN) {
        q_row0 = args.cu_q[bidx];
        k_row0 = args.cu_k[bidx];
        q_len = min(args.cu_q[bidx + 1] - q_row0, args.Nq);
        k_len = min(args.cu_k[bidx + 1] - k_row0, args.Nk);
        tma_b = 0;
    } else {
        q_row0 = 0;
        k_row0 = 0;
        q_len = args.Nq;
        k_len = args.Nk;
        tma_b = bidx;
    }
    if (q0 >= q_len) return;  // uniform over the CTA

    const int hk = h / args.group;
    const int last_q = min(q0 + 127, q_len - 1);
    const int kend = CAUSAL ? min(k_len, last_q + k_len - q_len + 1) : k_len;
    const int n_kv = kend > 0 ? (kend + 127) / 128 : 0;

    // Query row q (0-based in this sequence) is written iff it exists and, for
    // packed input, its token lies inside the caller's buffer.
    auto row_valid = [&](int q) -> bool {
        if (q >= q_len) return false;
        if constexpr (VARLEN) return q_row0 + q >= 0 && q_row0 + q < args.total_q;
        return true;
    };
    // Output addressing of query row q (0-based within this sequence).
    using T16 = uint16_t;
    T16* o_base = static_cast<T16*>(args.o);
    auto o_row = [&](int q) -> T16* {
        const size_t tok = VARLEN ? static_cast<size_t>(q_row0 + q) : static_cast<size_t>(bidx) * args.Nq + q;
        return o_base + (tok * args.Hq + h) * D;
    };
    auto lse_at = [&](int q) -> float* {
        if constexpr (VARLEN) {
            return args.lse + static_cast<size_t>(h) * args.total_q + q_row0 + q;
        } else {
            return args.lse + (static_cast<size_t>(bidx) * args.Hq + h) * args.Nq + q;
        }
    };

    if (n_kv == 0) {  // no row of this tile sees any key: O = 0, L = -inf
        if (threadIdx.x < 128) {
            const int q = q0 + static_cast<int>(threadIdx.x);
            if (row_valid(q)) {
                uint4* dst = reinterpret_cast<uint4*>(o_row(q));
#pragma unroll
                for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
                *lse_at(q) = -INFINITY;
            }
        }
        return;
    }

    uint8_t* sQ = smem + C::kQOff;
    uint8_t* sK = smem + C::kKOff;
    uint8_t* sV = smem + C::kVOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + S;
    uint64_t* v_full = k_empty + S;
    uint64_t* v_empty = v_full + S;
    uint64_t* s_full = v_empty + S;
    uint64_t* p_full = s_full + 2;
    uint64_t* o_done = p_full + 2;
    uint64_t* mma_final = o_done + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    int* abort_flag = reinterpret_cast<int*>(smem + C::kMiscOff + 4);

    const int warp = warp_id();
    const int lane = lane_id();

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < S; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 128);
        }
        mbar_init(o_done, 1);
        mbar_init(mma_final, 1);
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
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, C::kTileBytes);
#pragma unroll
            for (int s = 0; s < C::kSlabs; ++s)
                tma_load_4d(sQ + s * C::kSlabBytes, &tm_q, q_full, s * 64, h, q_row0 + q0, tma_b);
            int k_issued = 0, v_issued = 0;
            for (int j = 0; j < n_kv; ++j) {
                const int st = j % S;
                const uint32_t ph = (j / S) & 1;
                if (!mbar_wait(&k_empty[st], ph ^ 1u, wc, 1)) break;
                mbar_arrive_expect_tx(&k_full[st], C::kTileBytes);
#pragma unroll
                for (int s = 0; s < C::kSlabs; ++s)
                    tma_load_4d(sK + st * C::kTileBytes + s * C::kSlabBytes, &tm_k, &k_full[st], s * 64, hk,
                                k_row0 + j * 128, tma_b);
                ++k_issued;
                if (!mbar_wait(&v_empty[st], ph ^ 1u, wc, 2)) break;
                mbar_arrive_expect_tx(&v_full[st], C::kTileBytes);
#pragma unroll
                for (int s = 0; s < C::kSlabs; ++s)
                    tma_load_4d(sV + st * C::kTileBytes + s * C::kSlabBytes, &tm_v, &v_full[st], s * 64, hk,
                                k_row0 + j * 128, tma_b);
                ++v_issued;
            }
            // Drain: no TMA write may land after the CTA has exited.
            mbar_wait_drain(q_full, 0);
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
            bool ok = mbar_wait(q_full, 0, wc, 3);
            auto issue_s = [&](int j) -> bool {
                const int st = j % S;
                if (!mbar_wait(&k_full[st], (j / S) & 1, wc, 4)) return false;
                tc_fence_after();
                const uint32_t k_addr = smem_u32(sK + st * C::kTileBytes);
                const uint32_t d_col = tmem + ((j & 1) ? C::kColS1 : C::kColS0);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kSlabBytes + (kk & 3) * 32;
                    mma_ss(d_col, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024), id_qk,
                           kk > 0 ? 1u : 0u);
                }
                tc_commit(&k_empty[st]);
                tc_commit(&s_full[j & 1]);
                return true;
            };
            if (ok) ok = issue_s(0);
            if (ok && n_kv > 1) ok = issue_s(1);
            for (int j = 0; ok && j < n_kv; ++j) {
                const int st = j % S;
                if (!mbar_wait(&p_full[j & 1], (j >> 1) & 1, wc, 5)) break;
                if (!mbar_wait(&v_full[st], (j / S) & 1, wc, 6)) break;
                tc_fence_after();
                const uint32_t v_addr = smem_u32(sV + st * C::kTileBytes);
                const uint32_t p_col = tmem + ((j & 1) ? C::kColS1 : C::kColS0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    mma_ts(tmem + C::kColO, p_col + kk * 8, sdesc_sw128(v_addr + kk * 2048, C::kSlabBytes, 1024),
                           id_pv, (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&v_empty[st]);
                tc_commit(o_done);
                if (j + 2 < n_kv) {
                    // S_{j+2} overwrites the columns P_j is read from: let P_j V_j finish first
                    // (the ISA orders back-to-back MMAs only when they share the accumulator).
                    ok = mbar_wait(o_done, j & 1, wc, 10);
                    if (ok) ok = issue_s(j + 2);
                }
            }
            tc_commit(mma_final);
            mbar_wait_drain(mma_final, 0);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax / correction / epilogue
        const int w4 = warp & 3;
        const int r = w4 * 32 + lane;
        const int q = q0 + r;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(w4 * 32) << 16);
        const int row_limit = CAUSAL ? min(k_len, q + k_len - q_len + 1) : k_len;
        const float sl2 = args.scale_log2;
        float m = -INFINITY, l = 0.f, lr = 0.f;
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            ok = warp_all(mbar_wait(&s_full[j & 1], (j >> 1) & 1, wc, 7));
            if (!ok) break;
            tc_fence_after();
            const uint32_t s_addr = lane_base + ((j & 1) ? C::kColS1 : C::kColS0);
            uint32_t s[4][32];
            tmem_ld32(s_addr + 0, s[0]);
            tmem_ld32(s_addr + 32, s[1]);
            tmem_ld32(s_addr + 64, s[2]);
            tmem_ld32(s_addr + 96, s[3]);
            tmem_ld_wait(s[0]);
            tmem_ld_wait(s[1]);
            tmem_ld_wait(s[2]);
            tmem_ld_wait(s[3]);
            const int lim = row_limit - j * 128;  // columns >= lim are masked
            if (lim < 128) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c >= lim) s[c >> 5][c & 31] = __float_as_uint(-INFINITY);
            }
            // Row max as 16 independent partial maxima (a single chain of 128
            // dependent max operations would expose its whole latency).
            float mxp[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) mxp[i] = __uint_as_float(s[i >> 5][i & 31]);
#pragma unroll
            for (int c = 16; c < 128; ++c) mxp[c & 15] = fmaxf(mxp[c & 15], __uint_as_float(s[c >> 5][c & 31]));
#pragma unroll
            for (int w = 8; w > 0; w >>= 1)
#pragma unroll
                for (int i = 0; i < w; ++i) mxp[i] = fmaxf(mxp[i], mxp[i + w]);
            const float mx = mxp[0];
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
            // P is rounded to 16 bits for the P V product. l (exact fp32 sum)
            // gives L; lr, the sum of the ROUNDED values, normalises O, so the
            // weights applied to V sum to exactly one.
            float rsp[4] = {0.f, 0.f, 0.f, 0.f}, rsrp[4] = {0.f, 0.f, 0.f, 0.f};  // partial sums
            uint32_t pk[2][32];
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const float p0 = ex2_approx(fmaf(__uint_as_float(s[(2 * i) >> 5][(2 * i) & 31]), sl2, neg_m));
                const float p1 = ex2_approx(fmaf(__uint_as_float(s[(2 * i + 1) >> 5][(2 * i + 1) & 31]), sl2, neg_m));
                rsp[i & 3] += p0 + p1;
                const uint32_t u = pack2<BF16>(p0, p1);
                rsrp[i & 3] += unpack_lo<BF16>(u) + unpack_hi<BF16>(u);
                pk[i >> 5][i & 31] = u;
            }
            const float rs = (rsp[0] + rsp[1]) + (rsp[2] + rsp[3]);
            const float rsr = (rsrp[0] + rsrp[1]) + (rsrp[2] + rsrp[3]);
            l = l * alpha + rs;
            lr = lr * alpha + rsr;
            if (j > 0 && __any_sync(0xffffffffu, resc)) {
                ok = warp_all(mbar_wait(o_done, (j - 1) & 1, wc, 8));
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t ov[32];
                    tmem_ld32(lane_base + C::kColO + c0, ov);
                    tmem_ld_wait(ov);
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                    tmem_st32(lane_base + C::kColO + c0, ov);
                }
                tmem_st_wait();
            }
            tmem_st32(s_addr + 0, pk[0]);
            tmem_st32(s_addr + 32, pk[1]);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&p_full[j & 1]);
        }
        // The last two P V products may both be in flight here, more than one
        // phase of o_done apart, so the epilogue waits on the final commit.
        if (ok) ok = warp_all(mbar_wait(mma_final, 0, wc, 9));
        if (ok) {
            tc_fence_after();
            const bool row_ok = row_valid(q);
            const float inv_l = (lr > 0.f) ? 1.f / lr : 0.f;
            T16* dst = row_ok ? o_row(q) : nullptr;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t ov[32];
                tmem_ld32(lane_base + C::kColO + c0, ov);
                tmem_ld_wait(ov);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack2<BF16>(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
                if (row_ok) {
                    uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
                    for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
            if (row_ok) {
                float L;
                if (l > 0.f) {
                    float lg;
                    asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(l));
                    L = (m + lg) * kLn2;
                } else {
                    L = -INFINITY;
                }
                *lse_at(q) = L;
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
