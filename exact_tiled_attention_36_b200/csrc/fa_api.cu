// fa_api.cu: the C ABI of libfa.so (declared in include/fa.h).
//
// Host side only: argument validation, TMA descriptor encoding and kernel
// launches. Every step of the attention computation runs in the kernels of
// fa_fwd.cuh and fa_bwd.cuh; nothing here touches tensor data.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "bwd_grid.h"
#include "per_device.h"
#include "fa_fwd.cuh"
#include "fa_bwd.cuh"
#include "fa_bwd128.cuh"
#include "fa_decode.cuh"

namespace {

__device__ int g_fa_error = 0;  // first timeout site of any kernel (0 = none)
int g_last_site = 0;
cudaEvent_t g_bwd_ev_before = nullptr, g_bwd_ev_after = nullptr;  // fa_bwd_set_timing_events

constexpr float kLog2e = 1.4426950408889634074f;

PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Every argument of one tensor-map encoding (the key of the cache below). Built by
// memset + assignment, so the padding bytes are zero and memcmp compares keys.
struct MapKey {
    const void* base;
    int64_t rows, batches, sh, ss, sb;
    int d, H, box_h, box_rows, elem_bytes;
    int flags;  // bit 0: bf16, bit 1: 256-byte L2 promotion
};

// Encoded tensor maps of recent calls, per host thread (no lock): a caller that
// repeats a call with the same tensors and shapes, as a training or decoding loop
// does, reuses the maps instead of encoding them again. Direct-mapped on a hash of
// the key; a map is a pure function of its key, so a stale entry is never wrong,
// only replaced.
struct MapCache {
    static constexpr int kSlots = 128;
    MapKey key[kSlots];
    CUtensorMap map[kSlots];
    bool used[kSlots] = {};
};

uint32_t map_key_hash(const MapKey& k) {
    const unsigned char* p = reinterpret_cast<const unsigned char*>(&k);
    uint32_t h = 2166136261u;  // FNV-1a
    for (size_t i = 0; i < sizeof(MapKey); ++i) h = (h ^ p[i]) * 16777619u;
    return h;
}

fa_status encode_map(CUtensorMap* m, const MapKey& k);

// Tensor map of a [batches, rows, H, d] 16-bit tensor, box = box_rows rows x
// box_h heads x 64 columns, 128-byte swizzle. Rows past `rows` read as zero.
// 4-D map (d, H, rows, batches) over a tensor whose head, token and batch strides
// are sh, ss, sb elements (d contiguous); each stride must be a multiple of 16 bytes.
// `promote_256`: L2 promotion of each request to 256 bytes (else 128). A row of one
// head is 2 d bytes: with d = 64 the wider promotion also fetches the next head's row.
// `elem_bytes` = 1: one-byte elements (E4M3), a box of 128 columns (still 128 bytes).
fa_status make_map_box(CUtensorMap* m, const void* base, int d, int H, int64_t rows, int64_t batches, bool bf16,
                       int64_t sh, int64_t ss, int64_t sb, int box_h, int box_rows, bool promote_256 = true,
                       int elem_bytes = 2) {
    if (rows < 1) rows = 1;
    if (batches < 1) batches = 1;
    MapKey k;
    std::memset(&k, 0, sizeof(k));
    k.base = base;
    k.rows = rows;
    k.batches = batches;
    k.sh = sh;
    k.ss = ss;
    k.sb = sb;
    k.d = d;
    k.H = H;
    k.box_h = box_h;
    k.box_rows = box_rows;
    k.elem_bytes = elem_bytes;
    k.flags = (bf16 ? 1 : 0) | (promote_256 ? 2 : 0);
    thread_local MapCache cache;
    const int slot = static_cast<int>(map_key_hash(k) % MapCache::kSlots);
    if (cache.used[slot] && std::memcmp(&cache.key[slot], &k, sizeof(k)) == 0) {
        *m = cache.map[slot];
        return FA_OK;
    }
    const fa_status st = encode_map(m, k);
    if (st == FA_OK) {
        cache.key[slot] = k;
        cache.map[slot] = *m;
        cache.used[slot] = true;
    }
    return st;
}

fa_status encode_map(CUtensorMap* m, const MapKey& key) {
    auto enc = encode_tiled();
    if (!enc) return FA_ERR_CUDA;
    const void* base = key.base;
    const int d = key.d, H = key.H, box_h = key.box_h, box_rows = key.box_rows, elem_bytes = key.elem_bytes;
    const int64_t rows = key.rows, batches = key.batches, sh = key.sh, ss = key.ss, sb = key.sb;
    const bool bf16 = (key.flags & 1) != 0, promote_256 = (key.flags & 2) != 0;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(batches)};
    const cuuint64_t eb = static_cast<cuuint64_t>(elem_bytes);
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(sh) * eb, static_cast<cuuint64_t>(ss) * eb,
                                   static_cast<cuuint64_t>(sb) * eb};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / elem_bytes), static_cast<cuuint32_t>(box_h),
                               static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : (bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    CUresult r = enc(m, dt, 4,
                     const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B,
                     promote_256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// Box = 128 rows x 64 columns of one head (the attention kernels' K/V/Q tiles).
fa_status make_map_strided(CUtensorMap* m, const void* base, int d, int H, int64_t rows, int64_t batches, bool bf16,
                           int64_t sh, int64_t ss, int64_t sb) {
    return make_map_box(m, base, d, H, rows, batches, bf16, sh, ss, sb, 1, 128);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int current_device() {
    int dev = -1;
    return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
}

// Device address of the current device's error word (every GPU has its own copy
// of g_fa_error; a kernel must get the copy of the device it runs on). Null if
// the lookup fails.
int* error_word() {
    static fa::PerDevice<int*> ptrs;
    int* p = nullptr;
    ptrs.get(current_device(), [](int*& v) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_fa_error) != cudaSuccess || a == nullptr) return false;
        v = static_cast<int*>(a);
        return true;
    }, &p);
    return p;
}

// Streaming multiprocessors of the current device (the persistent forward runs at
// most one CTA per SM); 0 if the query fails.
int sm_count() {
    static fa::PerDevice<int> counts;
    const int dev = current_device();
    int n = 0;
    counts.get(dev, [dev](int& v) {
        return cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0;
    }, &n);
    return n;
}

// One-time set-up of a kernel on the current device: its dynamic shared memory
// limit raised to `smem` bytes, and the registers per thread it launches with.
// Returns that register count, or 0 if the set-up failed. `Kern` is the kernel
// itself, so each instantiation keeps its own per-device record.
template <auto Kern>
int kernel_setup(int smem) {
    static fa::PerDevice<int> regs;
    int n = 0;
    regs.get(current_device(), [smem](int& v) {
        if (cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return false;
        cudaFuncAttributes fa_attr{};
        if (cudaFuncGetAttributes(&fa_attr, Kern) != cudaSuccess || fa_attr.numRegs <= 0) return false;
        v = fa_attr.numRegs;
        return true;
    }, &n);
    return n;
}

// Units of 256 query rows for every (batch, head) and the persistent grid over them.
fa_status fwd_units(fa::FwdArgs& a, int nseq, int max_q, dim3& grid) {
    const long long nu = (static_cast<long long>(max_q) + 255) / 256;
    const long long n = nu * a.Hq * nseq;
    if (n > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    const int sms = sm_count();
    if (sms <= 0) return FA_ERR_CUDA;
    a.nu = static_cast<int>(nu);
    a.n_units = static_cast<int>(n);
    grid = dim3(static_cast<unsigned>(n < sms ? n : sms));
    return FA_OK;
}

fa_status common_checks(int Hq, int Hkv, int d, float scale, int causal, fa_dtype dtype) {
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
    if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_UNSUPPORTED;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (Hq > 65535) return FA_ERR_UNSUPPORTED;
    return FA_OK;
}

template <int D, bool BF16, int MASK, bool VARLEN, bool QKNORM, bool FP8 = false, bool KEYMASK = false>
fa_status launch_fwd_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fa::FwdArgs& a,
                       dim3 grid, cudaStream_t stream) {
    constexpr auto kern = fa::fa_fwd_kernel<D, BF16, MASK, VARLEN, QKNORM, FP8, KEYMASK>;
    constexpr int smem = fa::FwdCfg<D, FP8>::kSmemBytes;
    const int launch_regs = kernel_setup<kern>(smem);
    if (launch_regs == 0) return FA_ERR_CUDA;
    // The kernel moves registers between warpgroups with setmaxnreg; the split
    // must fit the pool the CTA is launched with, or the increase would wait
    // for registers that never come.
    if (launch_regs < fa::kFwdMinLaunchRegs) return FA_ERR_UNSUPPORTED;
    kern<<<grid, fa::kFwdThreads, smem, stream>>>(mq, mk, mv, a);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// The instantiations: mask none / causal / sliding window for plain inputs, fixed
// length and varlen; the window with global anchors for fixed length; QK
// normalisation for fixed length without a window; key masks for fixed length
// with mask none / causal.
template <int D, bool BF16>
fa_status launch_fwd_b(int mask, bool varlen, bool qknorm, const CUtensorMap& mq, const CUtensorMap& mk,
                       const CUtensorMap& mv, const fa::FwdArgs& a, dim3 grid, cudaStream_t s) {
    constexpr int N = fa::kMaskNone, C = fa::kMaskCausal, W = fa::kMaskWindow, A = fa::kMaskAnchor;
    if (a.key_bits != nullptr) {  // key masks: fixed length, no window, no normalisation
        if (qknorm || varlen || mask == W || mask == A) return FA_ERR_UNSUPPORTED;
        return mask == C ? launch_fwd_t<D, BF16, C, false, false, false, true>(mq, mk, mv, a, grid, s)
                         : launch_fwd_t<D, BF16, N, false, false, false, true>(mq, mk, mv, a, grid, s);
    }
    if (qknorm) {
        if (varlen || mask == W) return FA_ERR_UNSUPPORTED;
        return mask == C ? launch_fwd_t<D, BF16, C, false, true>(mq, mk, mv, a, grid, s)
                         : launch_fwd_t<D, BF16, N, false, true>(mq, mk, mv, a, grid, s);
    }
    if (mask == W) return varlen ? launch_fwd_t<D, BF16, W, true, false>(mq, mk, mv, a, grid, s)
                                 : launch_fwd_t<D, BF16, W, false, false>(mq, mk, mv, a, grid, s);
    if (mask == A) return varlen ? launch_fwd_t<D, BF16, A, true, false>(mq, mk, mv, a, grid, s)
                                 : launch_fwd_t<D, BF16, A, false, false>(mq, mk, mv, a, grid, s);
    if (mask == C) return varlen ? launch_fwd_t<D, BF16, C, true, false>(mq, mk, mv, a, grid, s)
                                 : launch_fwd_t<D, BF16, C, false, false>(mq, mk, mv, a, grid, s);
    return varlen ? launch_fwd_t<D, BF16, N, true, false>(mq, mk, mv, a, grid, s)
                  : launch_fwd_t<D, BF16, N, false, false>(mq, mk, mv, a, grid, s);
}

fa_status launch_fwd(int d, bool bf16, int mask, bool varlen, bool qknorm, const CUtensorMap& mq,
                     const CUtensorMap& mk, const CUtensorMap& mv, const fa::FwdArgs& a, dim3 grid, cudaStream_t s) {
    if (d == 64) return bf16 ? launch_fwd_b<64, true>(mask, varlen, qknorm, mq, mk, mv, a, grid, s)
                             : launch_fwd_b<64, false>(mask, varlen, qknorm, mq, mk, mv, a, grid, s);
    return bf16 ? launch_fwd_b<128, true>(mask, varlen, qknorm, mq, mk, mv, a, grid, s)
                : launch_fwd_b<128, false>(mask, varlen, qknorm, mq, mk, mv, a, grid, s);
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// keep [B, Nk] bytes (non-zero = visible) -> bits [B, words]: bit i of word w is key
// 32 w + i (zero past Nk).
__global__ void fa_pack_key_mask_kernel(const uint8_t* keep, uint32_t* bits, int B, int Nk, int words) {
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<long long>(B) * words) return;
    const long long b = idx / words;
    const int w = static_cast<int>(idx % words);
    uint32_t v = 0;
    for (int i = 0; i < 32; ++i) {
        const int key = 32 * w + i;
        if (key < Nk && keep[b * Nk + key]) v |= 1u << i;
    }
    bits[idx] = v;
}

// One CTA waits, with the kernels' bounded wait, on an mbarrier that nothing
// arrives on: the wait runs out, records the site and the kernel returns.
constexpr int kSelftestSite = 99;
__global__ void fa_selftest_wait_kernel(int* err) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        fa::mbar_init(&bar, 1);
        abort_flag = 0;
        fa::fence_mbar_init();
    }
    __syncthreads();
    const fa::WaitCtx wc{&abort_flag, err};
    fa::mbar_wait(&bar, 0, wc, kSelftestSite);
}

// d = 128 runs fa_bwd128_kernel (dQ^T = K^T dS^T with N = 128 queries); d = 64
// the single-tile kernel (its dQ^T would need M = 64, so it keeps dQ = dS K with
// M = 128 queries).
template <int D, bool BF16, bool CAUSAL, bool VARLEN>
fa_status launch_bwd_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                       const fa::BwdArgs& a, dim3 grid, cudaStream_t stream) {
    if constexpr (D == 128) {
        constexpr auto kern = fa::fa_bwd128_kernel<BF16, CAUSAL, VARLEN>;
        constexpr int smem = fa::Bwd128Cfg::kSmemBytes;
        const int launch_regs = kernel_setup<kern>(smem);
        if (launch_regs == 0) return FA_ERR_CUDA;
        // The kernel moves registers between warpgroups with setmaxnreg; the split
        // only fits if the launch holds enough registers per thread.
        if (launch_regs < fa::kBwd128MinLaunchRegs) return FA_ERR_UNSUPPORTED;
        kern<<<grid, fa::kBwd128Threads, smem, stream>>>(mq, mk, mv, mdo, a);
    } else {
        constexpr auto kern = fa::fa_bwd_kernel<D, BF16, CAUSAL, VARLEN>;
        constexpr int smem = fa::BwdCfg<D>::kSmemBytes;
        if (kernel_setup<kern>(smem) == 0) return FA_ERR_CUDA;
        kern<<<grid, fa::kBwdThreads, smem, stream>>>(mq, mk, mv, mdo, a);
    }
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, bool VARLEN>
fa_status launch_bwd_d(bool bf16, bool causal, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const CUtensorMap& mdo, const fa::BwdArgs& a, dim3 grid, cudaStream_t s) {
    if (bf16) return causal ? launch_bwd_t<D, true, true, VARLEN>(mq, mk, mv, mdo, a, grid, s)
                            : launch_bwd_t<D, true, false, VARLEN>(mq, mk, mv, mdo, a, grid, s);
    return causal ? launch_bwd_t<D, false, true, VARLEN>(mq, mk, mv, mdo, a, grid, s)
                  : launch_bwd_t<D, false, false, VARLEN>(mq, mk, mv, mdo, a, grid, s);
}

// Floats in the dQ accumulator: [B, Nq, Hq, 64] for d = 64; for d = 128 the
// queries of each (sequence, head) are padded to a multiple of four
// ([B, Hq, nq4, 128, 4]); varlen uses the same layout with B = num_seqs and
// Nq = max_seqlen_q.
size_t acc_floats(int B, int Hq, int Nq, int d) {
    if (d == 64) return static_cast<size_t>(B) * Hq * Nq * 64;
    return static_cast<size_t>(B) * Hq * ((static_cast<size_t>(Nq) + 3) / 4) * 512;
}

// The backward of fa_bwd and fa_varlen_bwd. Fixed length: nseq = B, rows = B * Nq,
// cu_q = cu_k = nullptr. Varlen: nseq = num_seqs, Nq / Nk the max_seqlen bounds,
// rows = total_q, and the maps span the packed buffers (total_q / total_k rows).
// Element strides of every tensor the backward reads or writes (batch, token, head).
struct BwdStrides {
    fa::Strides3 q, k, v, o, dout, dq, dk, dv;
};

// `causal` selects the masked kernels; their window is (wl, wr) (causal: (-1, 0)).
// `bs`: strided views (null: contiguous tensors).
fa_status bwd_common(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, void* workspace, int nseq, const int* cu_q,
                     const int* cu_k, int total_q, int total_k, int Hq, int Hkv, int Nq, int Nk, int d,
                     float scale, bool causal, bool bf16, cudaStream_t s, int wl = -1, int wr = 0,
                     int n_anchor = 0, const BwdStrides* bs = nullptr, const uint32_t* key_bits = nullptr) {
    const bool varlen = cu_q != nullptr;
    int* err = error_word();
    if (!err) return FA_ERR_CUDA;
    fa_status st;
    auto cont = [&](int rows_, int H) {
        return fa::Strides3{static_cast<long long>(rows_ > 0 ? rows_ : 1) * H * d, static_cast<long long>(H) * d, d};
    };
    BwdStrides def;
    def.q = def.o = def.dout = def.dq = cont(varlen ? total_q : Nq, Hq);
    def.k = def.v = def.dk = def.dv = cont(varlen ? total_k : Nk, Hkv);
    const BwdStrides& S = bs ? *bs : def;
    const size_t rows = static_cast<size_t>(varlen ? total_q : nseq * static_cast<size_t>(Nq)) * Hq;
    float* Dvec = static_cast<float*>(workspace);
    float* dq_acc = reinterpret_cast<float*>(static_cast<char*>(workspace) + round256(rows * sizeof(float)));
    const size_t acc_f4 = acc_floats(nseq, Hq, Nq, d) / 4;
    if (rows > 0) {
        const size_t threads = rows * (d / 8);
        const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
        // D = rowsum(dO o O) over [rows, d] viewed as one batch of rows / Hq tokens:
        // D lands in [Hq, tokens] = L's layout for varlen, [B, Hq, Nq] for fixed length.
        const int pb = varlen ? 1 : nseq, pn = varlen ? total_q : Nq;
        if (d == 64)
            fa::fa_bwd_preprocess<64><<<blocks, 256, 0, s>>>(static_cast<const uint16_t*>(o),
                                                             static_cast<const uint16_t*>(dout), Dvec, dq_acc, acc_f4,
                                                             pb, pn, Hq, bf16, S.o, S.dout);
        else
            fa::fa_bwd_preprocess<128><<<blocks, 256, 0, s>>>(static_cast<const uint16_t*>(o),
                                                              static_cast<const uint16_t*>(dout), Dvec, dq_acc,
                                                              acc_f4, pb, pn, Hq, bf16, S.o, S.dout);
        if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    const int kb = varlen ? 1 : nseq;
    const int kq_rows = varlen ? total_q : Nq, kk_rows = varlen ? total_k : Nk;
    if (kk_rows > 0 && Nk > 0) {
        CUtensorMap mq{}, mdo{}, mk, mv;
        if (kq_rows > 0 &&
            (st = make_map_strided(&mq, q, d, Hq, kq_rows, kb, bf16, S.q.h, S.q.s, S.q.b)) != FA_OK)
            return st;
        if (kq_rows > 0 &&
            (st = make_map_strided(&mdo, dout, d, Hq, kq_rows, kb, bf16, S.dout.h, S.dout.s, S.dout.b)) != FA_OK)
            return st;
        if ((st = make_map_strided(&mk, k, d, Hkv, kk_rows, kb, bf16, S.k.h, S.k.s, S.k.b)) != FA_OK) return st;
        if ((st = make_map_strided(&mv, v, d, Hkv, kk_rows, kb, bf16, S.v.h, S.v.s, S.v.b)) != FA_OK) return st;
        fa::BwdArgs a{};
        a.lse = lse;
        a.D = Dvec;
        a.dq_acc = dq_acc;
        a.nq4 = (Nq + 3) / 4;
        a.dk = dk;
        a.dv = dv;
        a.dk_sb = S.dk.b;
        a.dk_ss = S.dk.s;
        a.dk_sh = S.dk.h;
        a.dv_sb = S.dv.b;
        a.dv_ss = S.dv.s;
        a.dv_sh = S.dv.h;
        a.Hq = Hq;
        a.Hkv = Hkv;
        a.group = Hq / Hkv;
        a.Nq = Nq;
        a.Nk = Nk;
        a.cu_q = cu_q;
        a.cu_k = cu_k;
        a.total_q = total_q;
        a.scale = scale;
        a.scale_log2 = scale * kLog2e;
        a.wl = wl;
        a.wr = wr;
        a.n_anchor = n_anchor;
        a.key_bits = key_bits;
        a.kb_words = (Nk + 31) / 32;
        a.err = err;
        const unsigned nkt = static_cast<unsigned>((Nk + 127) / 128);
        if (nkt > 65535u) return FA_ERR_UNSUPPORTED;
        // One CTA per (sequence, KV head, key tile), in the order bwd_key_tile_fastest picks.
        const long long n_ctas = static_cast<long long>(nkt) * Hkv * nseq;
        const int sms = sm_count();
        if (sms <= 0) return FA_ERR_CUDA;
        a.kt_fast = fa::bwd_key_tile_fastest(causal, d, Hq, Hkv, n_anchor, n_ctas, sms) ? 1 : 0;
        const dim3 grid = (causal && !a.kt_fast) ? dim3(Hkv, nseq, nkt) : dim3(nkt, Hkv, nseq);
        const bool timed = g_bwd_ev_before && g_bwd_ev_after;
        if (timed && cudaEventRecord(g_bwd_ev_before, s) != cudaSuccess) return FA_ERR_CUDA;
        if (varlen)
            st = d == 64 ? launch_bwd_d<64, true>(bf16, causal, mq, mk, mv, mdo, a, grid, s)
                         : launch_bwd_d<128, true>(bf16, causal, mq, mk, mv, mdo, a, grid, s);
        else
            st = d == 64 ? launch_bwd_d<64, false>(bf16, causal, mq, mk, mv, mdo, a, grid, s)
                         : launch_bwd_d<128, false>(bf16, causal, mq, mk, mv, mdo, a, grid, s);
        if (st != FA_OK) return st;
        if (timed && cudaEventRecord(g_bwd_ev_after, s) != cudaSuccess) return FA_ERR_CUDA;
    }
    if (rows > 0) {
        if (d == 64) {
            // the accumulator's rows: [sequences, Nq (varlen: max_seqlen_q), Hq]
            const size_t n8 = static_cast<size_t>(nseq) * Nq * Hq * d / 8;
            fa::fa_bwd_dq_convert<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, s>>>(
                dq_acc, static_cast<uint16_t*>(dq), n8, scale, bf16, Nq, Hq, S.dq, cu_q);
        } else {
            const size_t n = static_cast<size_t>(nseq) * Hq * ((Nq + 3) / 4) * 64;
            fa::fa_bwd_dq_convert_g4<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(
                dq_acc, static_cast<uint16_t*>(dq), cu_q, nseq, Hq, Nq, (Nq + 3) / 4, scale, bf16, S.dq);
        }
        if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    return FA_OK;
}

// The argument checks of fa_bwd (nothing is launched when one fails).
fa_status bwd_checks(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                     float scale, int causal, fa_dtype dtype) {
    if (B < 1 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
    if ((Nq > 0 && (!q || !o || !lse || !dout || !dq)) || (Nk > 0 && (!k || !v || !dk || !dv)) || !workspace)
        return FA_ERR_INVALID_ARG;
    const fa_status st = common_checks(Hq, Hkv, d, scale, causal, dtype);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
        return FA_ERR_MISALIGNED;
    if (B > 65535 || Hkv > 65535) return FA_ERR_UNSUPPORTED;
    return FA_OK;
}

}  // namespace

extern "C" {

const char* fa_version(void) { return "0.1.0"; }

const char* fa_status_string(fa_status s) {
    switch (s) {
        case FA_OK: return "FA_OK";
        case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid argument";
        case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: unsupported head dim, dtype or size";
        case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED: tensor pointer or stride not 16-byte aligned";
        case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA call failed";
        case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a bounded device wait ran out";
    }
    return "unknown fa_status";
}

}  // extern "C" (reopened below)

namespace {

// Element strides of one 16-bit tensor: batch, token, head (d is contiguous).
struct Strides {
    long long b, s, h;
};

// Strides must be positive and multiples of 8 elements (16 bytes, the TMA rule).
fa_status check_strides(const Strides& t, bool with_batch) {
    if (t.s <= 0 || t.h <= 0 || (with_batch && t.b <= 0)) return FA_ERR_INVALID_ARG;
    if (t.s % 8 || t.h % 8 || (with_batch && t.b % 8)) return FA_ERR_MISALIGNED;
    return FA_OK;
}

// `causal` (0 or 1) is the caller's flag; a sliding window (wl, wr) other than the
// causal (-1, 0) or none (-1, -1) selects the window kernels instead.
fa_status fwd_fixed(const void* q, const void* k, const void* v, void* o, float* lse, Strides sq, Strides sk,
                    Strides sv, Strides so, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                    fa_dtype dtype, fa_stream_t stream, bool qknorm = false, float eps = 0.f,
                    bool validate_only = false, bool window = false, int wl = -1, int wr = 0,
                    int n_anchor = 0, const uint32_t* key_bits = nullptr) {
    if (B < 1 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
    if ((Nq > 0 && (!q || !o || !lse)) || (Nk > 0 && (!k || !v))) return FA_ERR_INVALID_ARG;
    fa_status st = common_checks(Hq, Hkv, d, scale, causal, dtype);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_MISALIGNED;
    for (const Strides* t : {&sq, &sk, &sv, &so})
        if ((st = check_strides(*t, true)) != FA_OK) return st;
    if (B > 65535) return FA_ERR_UNSUPPORTED;
    if (Nq == 0 || validate_only) return FA_OK;
    int* err = error_word();
    if (!err) return FA_ERR_CUDA;
    const bool bf16 = dtype == FA_BF16;
    CUtensorMap mq, mk{}, mv{};  // K/V maps stay unused (zero) when there is no key
    if ((st = make_map_strided(&mq, q, d, Hq, Nq, B, bf16, sq.h, sq.s, sq.b)) != FA_OK) return st;
    if (Nk > 0 && (st = make_map_strided(&mk, k, d, Hkv, Nk, B, bf16, sk.h, sk.s, sk.b)) != FA_OK) return st;
    if (Nk > 0 && (st = make_map_strided(&mv, v, d, Hkv, Nk, B, bf16, sv.h, sv.s, sv.b)) != FA_OK) return st;
    fa::FwdArgs a{};
    a.o = o;
    a.lse = lse;
    a.o_sb = so.b;
    a.o_ss = so.s;
    a.o_sh = so.h;
    a.wl = wl;
    a.wr = wr;
    a.n_anchor = n_anchor;
    a.key_bits = key_bits;
    a.kb_words = (Nk + 31) / 32;
    a.num_batches = B;
    a.Hq = Hq;
    a.group = Hq / Hkv;
    a.Nq = Nq;
    a.Nk = Nk;
    a.scale_log2 = scale * kLog2e;
    a.norm_eps = eps;
    a.err = err;
    dim3 grid;
    if ((st = fwd_units(a, B, Nq, grid)) != FA_OK) return st;
    const int mask = window ? (n_anchor > 0 ? fa::kMaskAnchor : fa::kMaskWindow)
                            : (causal ? fa::kMaskCausal : fa::kMaskNone);
    return launch_fwd(d, bf16, mask, false, qknorm, mq, mk, mv, a, grid, reinterpret_cast<cudaStream_t>(stream));
}

fa_status fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, Strides sq, Strides sk,
                     Strides sv, Strides so, const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                     int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv, int d,
                     float scale, int causal, fa_dtype dtype, fa_stream_t stream, bool window = false, int wl = -1,
                     int wr = 0, int n_anchor = 0) {
    if (num_seqs < 1 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0)
        return FA_ERR_INVALID_ARG;
    if (!cu_seqlens_q || !cu_seqlens_k || (total_q > 0 && (!q || !o || !lse)) || (total_k > 0 && (!k || !v)))
        return FA_ERR_INVALID_ARG;
    fa_status st = common_checks(Hq, Hkv, d, scale, causal, dtype);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
        return FA_ERR_MISALIGNED;
    for (const Strides* t : {&sq, &sk, &sv, &so})
        if ((st = check_strides(*t, false)) != FA_OK) return st;
    if (num_seqs > 65535) return FA_ERR_UNSUPPORTED;
    if (max_seqlen_q == 0 || total_q == 0) return FA_OK;
    int* err = error_word();
    if (!err) return FA_ERR_CUDA;
    const bool bf16 = dtype == FA_BF16;
    // The maps span exactly the caller's buffers: a tile that runs past the
    // last packed row reads zeros instead of memory beyond the allocation.
    CUtensorMap mq, mk{}, mv{};
    if ((st = make_map_strided(&mq, q, d, Hq, total_q, 1, bf16, sq.h, sq.s, sq.s * total_q)) != FA_OK) return st;
    if (total_k > 0 &&
        (st = make_map_strided(&mk, k, d, Hkv, total_k, 1, bf16, sk.h, sk.s, sk.s * total_k)) != FA_OK)
        return st;
    if (total_k > 0 &&
        (st = make_map_strided(&mv, v, d, Hkv, total_k, 1, bf16, sv.h, sv.s, sv.s * total_k)) != FA_OK)
        return st;
    fa::FwdArgs a{};
    a.o = o;
    a.lse = lse;
    a.o_sb = 0;
    a.o_ss = so.s;
    a.o_sh = so.h;
    a.wl = window ? wl : -1;
    a.wr = window ? wr : 0;
    a.n_anchor = window ? n_anchor : 0;
    a.cu_q = cu_seqlens_q;
    a.cu_k = cu_seqlens_k;
    a.num_batches = num_seqs;
    a.total_q = total_q;
    a.Hq = Hq;
    a.group = Hq / Hkv;
    a.Nq = max_seqlen_q;
    a.Nk = max_seqlen_k;
    a.scale_log2 = scale * kLog2e;
    a.err = err;
    dim3 grid;
    if ((st = fwd_units(a, num_seqs, max_seqlen_q, grid)) != FA_OK) return st;
    const int mask = window ? (a.n_anchor > 0 ? fa::kMaskAnchor : fa::kMaskWindow)
                            : (causal ? fa::kMaskCausal : fa::kMaskNone);
    return launch_fwd(d, bf16, mask, true, false, mq, mk, mv, a, grid, reinterpret_cast<cudaStream_t>(stream));
}

// The FP8 forward (fixed length, d = 128): E4M3 q, k, v with per-block factors.
fa_status fwd_fp8(const void* q, const void* k, const void* v, const float* q_scale, const float* k_scale,
                  const float* v_scale, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                  float scale, int causal, fa_stream_t stream) {
    if (B < 1 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
    if ((Nq > 0 && (!q || !o || !lse || !q_scale)) || (Nk > 0 && (!k || !v || !k_scale || !v_scale)))
        return FA_ERR_INVALID_ARG;
    fa_status st = common_checks(Hq, Hkv, d, scale, causal, FA_BF16);
    if (st != FA_OK) return st;
    if (d != 128) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
        (reinterpret_cast<uintptr_t>(q_scale) & 3u) || (reinterpret_cast<uintptr_t>(k_scale) & 3u) ||
        (reinterpret_cast<uintptr_t>(v_scale) & 3u))
        return FA_ERR_MISALIGNED;
    if (B > 65535) return FA_ERR_UNSUPPORTED;
    if (Nq == 0) return FA_OK;
    int* err = error_word();
    if (!err) return FA_ERR_CUDA;
    CUtensorMap mq, mk{}, mv{};
    const long long hq = static_cast<long long>(Hq) * d, hk = static_cast<long long>(Hkv) * d;
    if ((st = make_map_box(&mq, q, d, Hq, Nq, B, true, d, hq, hq * Nq, 1, 128, true, 1)) != FA_OK) return st;
    if (Nk > 0 && ((st = make_map_box(&mk, k, d, Hkv, Nk, B, true, d, hk, hk * Nk, 1, 128, true, 1)) != FA_OK ||
                   (st = make_map_box(&mv, v, d, Hkv, Nk, B, true, d, hk, hk * Nk, 1, 128, true, 1)) != FA_OK))
        return st;
    fa::FwdArgs a{};
    a.o = o;
    a.lse = lse;
    a.o_sb = static_cast<long long>(Nq) * Hq * d;
    a.o_ss = static_cast<long long>(Hq) * d;
    a.o_sh = d;
    a.wl = -1;
    a.wr = 0;
    a.num_batches = B;
    a.Hq = Hq;
    a.group = Hq / Hkv;
    a.Nq = Nq;
    a.Nk = Nk;
    a.scale_log2 = scale * kLog2e;
    a.q_scale = q_scale;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.nqb = (Nq + 127) / 128;
    a.nkb = (Nk + 127) / 128;
    a.err = err;
    dim3 grid;
    if ((st = fwd_units(a, B, Nq, grid)) != FA_OK) return st;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return causal ? launch_fwd_t<128, true, fa::kMaskCausal, false, false, true>(mq, mk, mv, a, grid, s)
                  : launch_fwd_t<128, true, fa::kMaskNone, false, false, true>(mq, mk, mv, a, grid, s);
}

Strides contiguous(int rows, int H, int d) {
    return {static_cast<long long>(rows > 0 ? rows : 1) * H * d, static_cast<long long>(H) * d, d};
}

fa_status read_strides(const long long* p, bool with_batch, Strides* out) {
    if (!p) return FA_ERR_INVALID_ARG;
    *out = with_batch ? Strides{p[0], p[1], p[2]} : Strides{0, p[0], p[1]};
    return FA_OK;
}

// ---------------------------------------------------------------- decode
// Row layout of the decode tile: nb blocks of gh heads, one block per 32 TMEM
// lanes, when the group splits so (the exponentials then spread over the four
// softmax warps); else one block of all g heads in lanes 0 .. g Nq - 1.
void dec_layout(int g, int Nq, int& nb, int& gh) {
    for (int k : {4, 2})
        if (g % k == 0 && (g / k) * Nq <= 32) {
            nb = k;
            gh = g / k;
            return;
        }
    nb = 1;
    gh = g;
}

constexpr int kDecMaxCtas = 1024;

// CTAs the split kernel may use on the current device (0 without one).
int dec_max_ctas() {
    const int sms = sm_count();
    return sms < kDecMaxCtas ? sms : kDecMaxCtas;
}

// Workspace of the decode: meta (T and each item's first tile, int64), then the
// partial L (fp32 [slots, R]) and O (fp32 [slots, R, d]), each 256-byte aligned;
// slots = CTAs + items (the slot of CTA c's segment of item i is c + i).
struct DecWs {
    size_t meta, lse, total;
};

bool dec_ws(int B, int Hq, int Hkv, int Nq, int d, DecWs& w) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Nq < 0 || (d != 64 && d != 128)) return false;
    const long long R = static_cast<long long>(Hq / Hkv) * Nq;
    if (R > 128) return false;
    const int G = dec_max_ctas();
    if (G <= 0) return false;
    const size_t items = static_cast<size_t>(B) * Hkv;
    const size_t slots = items + G;
    // d = 64 may pair KV heads: half the items with twice the rows (bounded by this).
    const size_t rows = d == 64 ? 2 * R : R;
    w.meta = round256((1 + items) * sizeof(long long));
    w.lse = round256(slots * rows * sizeof(float));
    w.total = w.meta + w.lse + round256(slots * rows * d * sizeof(float));
    return true;
}

// RN = 0: the row-per-lane kernel (any R <= 128); RN = 16 or 32: the narrow kernel
// with the products' operands swapped (R <= RN).
// PAIR (d = 64, narrow only): the split kernel runs as d = 128 over pairs of KV heads;
// the merge writes d = 64.
template <int D, bool BF16, bool SEQLENS, bool PAGED, int RN, bool PAIR = false>
fa_status launch_dec_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fa::DecodeArgs& a,
                       int causal, bool run_split, cudaStream_t s) {
    static_assert(!PAIR || (D == 64 && RN != 0), "paired KV heads: d = 64, narrow kernel");
    constexpr int DK = PAIR ? 128 : D;
    if (run_split) {
        if constexpr (RN == 0) {
            constexpr auto kern = fa::fa_decode_kernel<D, BF16, SEQLENS, PAGED>;
            constexpr int smem = fa::DecCfg<D>::kSmemBytes;
            if (kernel_setup<kern>(smem) == 0) return FA_ERR_CUDA;
            kern<<<a.G, fa::kDecThreads, smem, s>>>(mq, mk, mv, a, causal);
        } else {
            constexpr auto kern = fa::fa_decode_narrow_kernel<DK, BF16, SEQLENS, PAGED, RN>;
            constexpr int smem = fa::DecNarrowCfg<DK, RN>::kSmemBytes;
            if (kernel_setup<kern>(smem) == 0) return FA_ERR_CUDA;
            kern<<<a.G, fa::kDecThreads, smem, s>>>(mq, mk, mv, a, causal);
        }
        if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    // The merge launches as a programmatic dependent of the split kernel, so its
    // launch overlaps the split kernel's tail; it waits for the split kernel's
    // results in the kernel (griddepcontrol.wait).
    const long long rows = static_cast<long long>(a.B) * a.Hkv * a.R;  // one block per (item, row)
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(rows));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = run_split ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, fa::fa_decode_combine<D, BF16, SEQLENS>, a) != cudaSuccess) return FA_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, bool BF16, int RN, bool PAIR>
fa_status launch_dec_r(bool seqlens, bool paged, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const fa::DecodeArgs& a, int causal, bool run_split, cudaStream_t s) {
    if (paged) return launch_dec_t<D, BF16, true, true, RN, PAIR>(mq, mk, mv, a, causal, run_split, s);
    if (seqlens) return launch_dec_t<D, BF16, true, false, RN, PAIR>(mq, mk, mv, a, causal, run_split, s);
    return launch_dec_t<D, BF16, false, false, RN, PAIR>(mq, mk, mv, a, causal, run_split, s);
}

template <int D, bool BF16>
fa_status launch_dec_b(int rn, bool pair, bool seqlens, bool paged, const CUtensorMap& mq, const CUtensorMap& mk,
                       const CUtensorMap& mv, const fa::DecodeArgs& a, int causal, bool run_split, cudaStream_t s) {
    if constexpr (D == 64) {
        if (pair) return rn == 16 ? launch_dec_r<64, BF16, 16, true>(seqlens, paged, mq, mk, mv, a, causal, run_split, s)
                                  : launch_dec_r<64, BF16, 32, true>(seqlens, paged, mq, mk, mv, a, causal, run_split, s);
    }
    if (rn == 16) return launch_dec_r<D, BF16, 16, false>(seqlens, paged, mq, mk, mv, a, causal, run_split, s);
    if (rn == 32) return launch_dec_r<D, BF16, 32, false>(seqlens, paged, mq, mk, mv, a, causal, run_split, s);
    return launch_dec_r<D, BF16, 0, false>(seqlens, paged, mq, mk, mv, a, causal, run_split, s);
}

// fa_decode (paged = false: k, v [B, Nk, Hkv, d]) and fa_decode_paged (k, v page
// pools [num_pages, page_size, Hkv, d] through block_table [B, max_pages]).
fa_status decode_common(const void* q, const void* k, const void* v, void* o, float* lse, const int* seqlens,
                        const int* block_table, void* workspace, int B, int Hq, int Hkv, int Nq, int Nk,
                        bool paged, int num_pages, int page_size, int max_pages, int d, float scale, int causal,
                        fa_dtype dtype, fa_stream_t stream) {
    if (B < 1 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
    fa_status st = common_checks(Hq, Hkv, d, scale, causal, dtype);
    if (st != FA_OK) return st;
    if (paged) {
        if (!seqlens || !block_table || num_pages < 1 || max_pages < 1 || page_size < 16) return FA_ERR_INVALID_ARG;
        if (!(page_size == 16 || page_size == 32 || page_size % 64 == 0)) return FA_ERR_UNSUPPORTED;
    }
    const int cap = paged ? (static_cast<long long>(max_pages) * page_size > 0x7fffffffLL ? -1 : max_pages * page_size)
                          : Nk;
    if (cap < 0) return FA_ERR_UNSUPPORTED;
    if (Nq > 0 && (!q || !o || !lse || !workspace)) return FA_ERR_INVALID_ARG;
    if (cap > 0 && (!k || !v)) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
        !aligned16(workspace) || (reinterpret_cast<uintptr_t>(seqlens) & 3u) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3u))
        return FA_ERR_MISALIGNED;
    const int g = Hq / Hkv;
    if (static_cast<long long>(g) * Nq > 128) return FA_ERR_UNSUPPORTED;  // one tile holds a group's queries
    const long long items = static_cast<long long>(B) * Hkv;
    const long long max_tiles = items * ((static_cast<long long>(cap) + 127) / 128);
    if (items * g * Nq > 0x7fffffffLL || max_tiles > (1LL << 40) || B > 65535 || Nq > 65535)
        return FA_ERR_UNSUPPORTED;
    if (Nq == 0) return FA_OK;
    int* err = error_word();
    if (!err) return FA_ERR_CUDA;
    DecWs w;
    if (!dec_ws(B, Hq, Hkv, Nq, d, w)) return FA_ERR_CUDA;
    const bool bf16 = dtype == FA_BF16;
    // Up to 32 rows: the narrow kernel (one box of all g heads x Nq tokens); more:
    // the row-per-lane kernel with its lane layout.
    const int R = g * Nq;
    // d = 64, even Hkv, R <= 16: pairs of KV heads (256-byte K/V rows), 2 roundup8(R)
    // tile rows.
    const bool pair = d == 64 && Hkv % 2 == 0 && R <= 16;
    const int r8 = (R + 7) / 8 * 8;
    const int rows = pair ? 2 * r8 : R;
    const int rn = rows <= 16 ? 16 : (rows <= 32 ? 32 : 0);
    int nb = 1, gh = g;
    if (rn == 0) dec_layout(g, Nq, nb, gh);
    CUtensorMap mq, mk{}, mv{};
    const long long hd = static_cast<long long>(Hq) * d;
    if ((st = make_map_box(&mq, q, d, Hq, Nq, B, bf16, d, hd, hd * Nq, gh, Nq)) != FA_OK) return st;
    const int page_box = page_size < 64 ? page_size : 64;
    if (cap > 0) {
        const long long kd = static_cast<long long>(Hkv) * d;
        // Paired heads: the caches seen as Hkv / 2 heads of 128 values (the same memory).
        const int md = pair ? 128 : d, mh = pair ? Hkv / 2 : Hkv;
        // Each K/V row of a head is read once: the L2 request stays at one head's row.
        const bool p256 = md == 128;
        if (paged) {
            if ((st = make_map_box(&mk, k, md, mh, page_size, num_pages, bf16, md, kd, kd * page_size, 1, page_box,
                                   p256)) != FA_OK ||
                (st = make_map_box(&mv, v, md, mh, page_size, num_pages, bf16, md, kd, kd * page_size, 1, page_box,
                                   p256)) != FA_OK)
                return st;
        } else if ((st = make_map_box(&mk, k, md, mh, Nk, B, bf16, md, kd, kd * Nk, 1, 128, p256)) != FA_OK ||
                   (st = make_map_box(&mv, v, md, mh, Nk, B, bf16, md, kd, kd * Nk, 1, 128, p256)) != FA_OK) {
            return st;
        }
    }
    fa::DecodeArgs a{};
    a.o = o;
    a.lse = lse;
    a.meta = static_cast<long long*>(workspace);
    a.lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + w.meta);
    a.o_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + w.meta + w.lse);
    a.seqlens = seqlens;
    a.block_table = block_table;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = pair ? Hkv / 2 : Hkv;  // items per sequence
    a.group = g;
    a.Nq = Nq;
    a.Nk = paged ? cap : Nk;
    a.R = pair ? 2 * R : R;  // rows per item
    a.pair = pair ? 1 : 0;
    a.rg = R;
    a.r8 = pair ? r8 : 0;
    a.cap = cap;
    a.page_size = page_size;
    a.max_pages = max_pages;
    a.page_box = page_box;
    a.nb = nb;
    a.gh = gh;
    a.scale_log2 = scale * kLog2e;
    a.err = err;
    // Fixed lengths: exactly T tiles; with lengths, at most T tiles (each CTA finds
    // its share of the true T itself).
    const int sms = dec_max_ctas();
    const long long item_tiles = pair ? max_tiles / 2 : max_tiles;  // paired items hold two heads' tiles
    a.G = static_cast<int>(item_tiles < sms ? item_tiles : sms);
    const bool run_split = max_tiles > 0;
    if (a.G < 1) a.G = 1;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool sl = seqlens != nullptr;
    if (d == 64) return bf16 ? launch_dec_b<64, true>(rn, pair, sl, paged, mq, mk, mv, a, causal, run_split, s)
                             : launch_dec_b<64, false>(rn, pair, sl, paged, mq, mk, mv, a, causal, run_split, s);
    return bf16 ? launch_dec_b<128, true>(rn, false, sl, paged, mq, mk, mv, a, causal, run_split, s)
                : launch_dec_b<128, false>(rn, false, sl, paged, mq, mk, mv, a, causal, run_split, s);
}

// The backward of fa_varlen_bwd / fa_varlen_bwd_window(_anchor); the masked kernels
// take the window (wl, wr) (causal: (-1, 0)) and the anchor keys of every sequence.
fa_status varlen_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, void* workspace, const int* cu_seqlens_q,
                     const int* cu_seqlens_k, int num_seqs, int total_q, int total_k, int max_seqlen_q,
                     int max_seqlen_k, int Hq, int Hkv, int d, float scale, int causal, fa_dtype dtype,
                     fa_stream_t stream, int wl = -1, int wr = 0, int n_anchor = 0,
                     const BwdStrides* bs = nullptr) {
    if (num_seqs < 1 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0)
        return FA_ERR_INVALID_ARG;
    if (!cu_seqlens_q || !cu_seqlens_k || !workspace || (total_q > 0 && (!q || !o || !lse || !dout || !dq)) ||
        (total_k > 0 && (!k || !v || !dk || !dv)))
        return FA_ERR_INVALID_ARG;
    fa_status st = common_checks(Hq, Hkv, d, scale, causal, dtype);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
        return FA_ERR_MISALIGNED;
    if (num_seqs > 65535 || Hkv > 65535) return FA_ERR_UNSUPPORTED;
    return bwd_common(q, k, v, o, lse, dout, dq, dk, dv, workspace, num_seqs, cu_seqlens_q, cu_seqlens_k, total_q,
                      total_k, Hq, Hkv, max_seqlen_q, max_seqlen_k, d, scale, causal != 0, dtype == FA_BF16,
                      reinterpret_cast<cudaStream_t>(stream), wl, wr, n_anchor, bs);
}

}  // namespace

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                 int Nq, int Nk, int d, float scale, int causal, fa_dtype dtype, fa_stream_t stream) {
    return fwd_fixed(q, k, v, o, lse, contiguous(Nq, Hq, d), contiguous(Nk, Hkv, d), contiguous(Nk, Hkv, d),
                     contiguous(Nq, Hq, d), B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, stream);
}

size_t fa_fwd_qk_rmsnorm_workspace_size(int B, int Nk, int Hkv, int d) {
    if (B < 1 || Nk < 0 || Hkv < 1 || (d != 64 && d != 128)) return 0;
    return round256(static_cast<size_t>(B) * Nk * Hkv * d * 2);
}

fa_status fa_fwd_qk_rmsnorm(const void* q, const void* k, const void* v, void* o, float* lse, void* workspace,
                            int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, float eps,
                            fa_dtype dtype, fa_stream_t stream) {
    if (!(std::isfinite(eps) && eps >= 0.f)) return FA_ERR_INVALID_ARG;
    if (Nk > 0 && !workspace) return FA_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
    // Everything fa_fwd checks, before anything runs (on the real K: the normalised
    // copy has its layout).
    fa_status st = fwd_fixed(q, k, v, o, lse, contiguous(Nq, Hq, d), contiguous(Nk, Hkv, d),
                             contiguous(Nk, Hkv, d), contiguous(Nq, Hq, d), B, Hq, Hkv, Nq, Nk, d, scale, causal,
                             dtype, stream, true, eps, /*validate_only=*/true);
    if (st != FA_OK || Nq == 0) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t rows = static_cast<size_t>(B) * Nk * Hkv;
    if (rows > 0) {
        const size_t threads = rows * (d / 8);
        const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
        const uint16_t* kx = static_cast<const uint16_t*>(k);
        uint16_t* ky = static_cast<uint16_t*>(workspace);
        if (d == 64)
            dtype == FA_BF16 ? fa::fa_rms_normalise_rows<64, true><<<blocks, 256, 0, s>>>(kx, ky, rows, eps)
                             : fa::fa_rms_normalise_rows<64, false><<<blocks, 256, 0, s>>>(kx, ky, rows, eps);
        else
            dtype == FA_BF16 ? fa::fa_rms_normalise_rows<128, true><<<blocks, 256, 0, s>>>(kx, ky, rows, eps)
                             : fa::fa_rms_normalise_rows<128, false><<<blocks, 256, 0, s>>>(kx, ky, rows, eps);
        if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    return fwd_fixed(q, Nk > 0 ? workspace : k, v, o, lse, contiguous(Nq, Hq, d), contiguous(Nk, Hkv, d),
                     contiguous(Nk, Hkv, d), contiguous(Nq, Hq, d), B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype,
                     stream, true, eps);
}

fa_status fa_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                        int Nq, int Nk, int d, float scale, int window_left, int window_right, fa_dtype dtype,
                        fa_stream_t stream) {
    const int wl = window_left < 0 ? -1 : window_left, wr = window_right < 0 ? -1 : window_right;
    const bool none = wl < 0 && wr < 0, causal = wl < 0 && wr == 0;
    return fwd_fixed(q, k, v, o, lse, contiguous(Nq, Hq, d), contiguous(Nk, Hkv, d), contiguous(Nk, Hkv, d),
                     contiguous(Nq, Hq, d), B, Hq, Hkv, Nq, Nk, d, scale, causal ? 1 : 0, dtype, stream, false, 0.f,
                     false, !none && !causal, wl, wr);
}

fa_status fa_fwd_window_anchor(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                               int Hkv, int Nq, int Nk, int d, float scale, int window_left, int window_right,
                               int n_anchor, fa_dtype dtype, fa_stream_t stream) {
    if (n_anchor < 0) return FA_ERR_INVALID_ARG;
    const int wl = window_left < 0 ? -1 : window_left, wr = window_right < 0 ? -1 : window_right;
    if (n_anchor == 0 || wl < 0)  // no anchors, or nothing below the window to add
        return fa_fwd_window(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, wl, wr, dtype, stream);
    return fwd_fixed(q, k, v, o, lse, contiguous(Nq, Hq, d), contiguous(Nk, Hkv, d), contiguous(Nk, Hkv, d),
                     contiguous(Nq, Hq, d), B, Hq, Hkv, Nq, Nk, d, scale, 0, dtype, stream, false, 0.f, false, true,
                     wl, wr, n_anchor);
}

fa_status fa_pack_key_mask(const unsigned char* keep, unsigned int* key_bits, int B, int Nk, fa_stream_t stream) {
    if (B < 1 || Nk < 0 || (Nk > 0 && (!keep || !key_bits))) return FA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(key_bits) & 3u) return FA_ERR_MISALIGNED;
    const int words = (Nk + 31) / 32;
    const long long n = static_cast<long long>(B) * words;
    if (n == 0) return FA_OK;
    fa_pack_key_mask_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        keep, key_bits, B, Nk, words);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_fwd_keymask(const void* q, const void* k, const void* v, void* o, float* lse,
                         const unsigned int* key_bits, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                         int causal, fa_dtype dtype, fa_stream_t stream) {
    if (Nk > 0 && !key_bits) return FA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(key_bits) & 3u) return FA_ERR_MISALIGNED;
    return fwd_fixed(q, k, v, o, lse, contiguous(Nq, Hq, d), contiguous(Nk, Hkv, d), contiguous(Nk, Hkv, d),
                     contiguous(Nq, Hq, d), B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, stream, false, 0.f, false,
                     false, -1, 0, 0, key_bits);
}

fa_status fa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                         const long long* q_strides, const long long* k_strides, const long long* v_strides,
                         const long long* o_strides, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                         int causal, fa_dtype dtype, fa_stream_t stream) {
    Strides sq, sk, sv, so;
    fa_status st;
    if ((st = read_strides(q_strides, true, &sq)) != FA_OK || (st = read_strides(k_strides, true, &sk)) != FA_OK ||
        (st = read_strides(v_strides, true, &sv)) != FA_OK || (st = read_strides(o_strides, true, &so)) != FA_OK)
        return st;
    return fwd_fixed(q, k, v, o, lse, sq, sk, sv, so, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, stream);
}

fa_status fa_varlen_fwd(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens_q,
                        const int* cu_seqlens_k, int num_seqs, int total_q, int total_k, int max_seqlen_q,
                        int max_seqlen_k, int Hq, int Hkv, int d, float scale, int causal, fa_dtype dtype,
                        fa_stream_t stream) {
    return fwd_varlen(q, k, v, o, lse, contiguous(total_q, Hq, d), contiguous(total_k, Hkv, d),
                      contiguous(total_k, Hkv, d), contiguous(total_q, Hq, d), cu_seqlens_q, cu_seqlens_k, num_seqs,
                      total_q, total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, causal, dtype, stream);
}

fa_status fa_varlen_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                                const long long* q_strides, const long long* k_strides,
                                const long long* v_strides, const long long* o_strides, const int* cu_seqlens_q,
                                const int* cu_seqlens_k, int num_seqs, int total_q, int total_k, int max_seqlen_q,
                                int max_seqlen_k, int Hq, int Hkv, int d, float scale, int causal, fa_dtype dtype,
                                fa_stream_t stream) {
    Strides sq, sk, sv, so;
    fa_status st;
    if ((st = read_strides(q_strides, false, &sq)) != FA_OK || (st = read_strides(k_strides, false, &sk)) != FA_OK ||
        (st = read_strides(v_strides, false, &sv)) != FA_OK || (st = read_strides(o_strides, false, &so)) != FA_OK)
        return st;
    return fwd_varlen(q, k, v, o, lse, sq, sk, sv, so, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q, total_k,
                      max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, causal, dtype, stream);
}

size_t fa_bwd_workspace_size(int B, int Hq, int Nq, int d) {
    if (B < 1 || Hq < 1 || Nq < 0 || (d != 64 && d != 128)) return 0;
    const size_t rows = static_cast<size_t>(B) * Hq * Nq;
    return round256(rows * sizeof(float)) + round256(acc_floats(B, Hq, Nq, d) * sizeof(float));
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                 void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                 float scale, int causal, fa_dtype dtype, fa_stream_t stream) {
    const fa_status st = bwd_checks(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                                    dtype);
    if (st != FA_OK) return st;
    return bwd_common(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, nullptr, nullptr, 0, 0, Hq, Hkv, Nq, Nk, d,
                      scale, causal != 0, dtype == FA_BF16, reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_bwd_window(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv,
                        int Nq, int Nk, int d, float scale, int window_left, int window_right, fa_dtype dtype,
                        fa_stream_t stream) {
    const int wl = window_left < 0 ? -1 : window_left, wr = window_right < 0 ? -1 : window_right;
    const bool masked = wl >= 0 || wr >= 0;
    const fa_status st = bwd_checks(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, scale,
                                    masked ? 1 : 0, dtype);
    if (st != FA_OK) return st;
    return bwd_common(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, nullptr, nullptr, 0, 0, Hq, Hkv, Nq, Nk, d,
                      scale, masked, dtype == FA_BF16, reinterpret_cast<cudaStream_t>(stream), wl, wr);
}

fa_status fa_bwd_window_anchor(const void* q, const void* k, const void* v, const void* o, const float* lse,
                               const void* dout, void* dq, void* dk, void* dv, void* workspace, int B, int Hq,
                               int Hkv, int Nq, int Nk, int d, float scale, int window_left, int window_right,
                               int n_anchor, fa_dtype dtype, fa_stream_t stream) {
    if (n_anchor < 0) return FA_ERR_INVALID_ARG;
    const int wl = window_left < 0 ? -1 : window_left, wr = window_right < 0 ? -1 : window_right;
    const bool masked = wl >= 0 || wr >= 0;
    const fa_status st = bwd_checks(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, scale,
                                    masked ? 1 : 0, dtype);
    if (st != FA_OK) return st;
    return bwd_common(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, nullptr, nullptr, 0, 0, Hq, Hkv, Nq, Nk, d,
                      scale, masked, dtype == FA_BF16, reinterpret_cast<cudaStream_t>(stream), wl, wr,
                      wl >= 0 ? n_anchor : 0);
}

fa_status fa_bwd_strided(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, void* workspace,
                         const long long* q_strides, const long long* k_strides, const long long* v_strides,
                         const long long* o_strides, const long long* do_strides, const long long* dq_strides,
                         const long long* dk_strides, const long long* dv_strides, int B, int Hq, int Hkv, int Nq,
                         int Nk, int d, float scale, int causal, fa_dtype dtype, fa_stream_t stream) {
    const long long* given[8] = {q_strides, k_strides, v_strides, o_strides, do_strides, dq_strides, dk_strides,
                                 dv_strides};
    Strides t[8];
    fa_status st;
    for (int i = 0; i < 8; ++i) {
        if ((st = read_strides(given[i], true, &t[i])) != FA_OK) return st;
        if ((st = check_strides(t[i], true)) != FA_OK) return st;
    }
    st = bwd_checks(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype);
    if (st != FA_OK) return st;
    auto s3 = [](const Strides& x) { return fa::Strides3{x.b, x.s, x.h}; };
    const BwdStrides bs{s3(t[0]), s3(t[1]), s3(t[2]), s3(t[3]), s3(t[4]), s3(t[5]), s3(t[6]), s3(t[7])};
    return bwd_common(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, nullptr, nullptr, 0, 0, Hq, Hkv, Nq, Nk, d,
                      scale, causal != 0, dtype == FA_BF16, reinterpret_cast<cudaStream_t>(stream), -1, 0, 0, &bs);
}

fa_status fa_bwd_keymask(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, void* workspace,
                         const unsigned int* key_bits, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                         int causal, fa_dtype dtype, fa_stream_t stream) {
    if (Nk > 0 && !key_bits) return FA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(key_bits) & 3u) return FA_ERR_MISALIGNED;
    const fa_status st = bwd_checks(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                                    dtype);
    if (st != FA_OK) return st;
    return bwd_common(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, nullptr, nullptr, 0, 0, Hq, Hkv, Nq, Nk, d,
                      scale, causal != 0, dtype == FA_BF16, reinterpret_cast<cudaStream_t>(stream), -1, 0, 0, nullptr,
                      key_bits);
}

size_t fa_varlen_bwd_workspace_size(int num_seqs, int total_q, int max_seqlen_q, int Hq, int d) {
    if (num_seqs < 1 || total_q < 0 || max_seqlen_q < 0 || Hq < 1 || (d != 64 && d != 128)) return 0;
    const size_t rows = static_cast<size_t>(total_q) * Hq;
    return round256(rows * sizeof(float)) + round256(acc_floats(num_seqs, Hq, max_seqlen_q, d) * sizeof(float));
}

fa_status fa_varlen_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, void* workspace, const int* cu_seqlens_q,
                        const int* cu_seqlens_k, int num_seqs, int total_q, int total_k, int max_seqlen_q,
                        int max_seqlen_k, int Hq, int Hkv, int d, float scale, int causal, fa_dtype dtype,
                        fa_stream_t stream) {
    return varlen_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q,
                      total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, causal, dtype, stream);
}

fa_status fa_varlen_bwd_strided(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                const void* dout, void* dq, void* dk, void* dv, void* workspace,
                                const long long* q_strides, const long long* k_strides, const long long* v_strides,
                                const long long* o_strides, const long long* do_strides,
                                const long long* dq_strides, const long long* dk_strides,
                                const long long* dv_strides, const int* cu_seqlens_q, const int* cu_seqlens_k,
                                int num_seqs, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int Hq,
                                int Hkv, int d, float scale, int causal, fa_dtype dtype, fa_stream_t stream) {
    const long long* given[8] = {q_strides, k_strides, v_strides, o_strides, do_strides, dq_strides, dk_strides,
                                 dv_strides};
    Strides t[8];
    fa_status st;
    for (int i = 0; i < 8; ++i) {
        if ((st = read_strides(given[i], false, &t[i])) != FA_OK) return st;
        if ((st = check_strides(t[i], false)) != FA_OK) return st;
    }
    // One "batch" of all packed rows: its stride only sizes the TMA maps' last dimension.
    auto s3 = [](const Strides& x, int rows) {
        return fa::Strides3{x.s * static_cast<long long>(rows > 0 ? rows : 1), x.s, x.h};
    };
    const BwdStrides bs{s3(t[0], total_q), s3(t[1], total_k), s3(t[2], total_k), s3(t[3], total_q),
                        s3(t[4], total_q), s3(t[5], total_q), s3(t[6], total_k), s3(t[7], total_k)};
    return varlen_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q,
                      total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, causal, dtype, stream, -1, 0, 0, &bs);
}

fa_status fa_varlen_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse,
                               const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs, int total_q,
                               int total_k, int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv, int d, float scale,
                               int window_left, int window_right, fa_dtype dtype, fa_stream_t stream) {
    const int wl = window_left < 0 ? -1 : window_left, wr = window_right < 0 ? -1 : window_right;
    const bool none = wl < 0 && wr < 0, causal = wl < 0 && wr == 0;
    return fwd_varlen(q, k, v, o, lse, contiguous(total_q, Hq, d), contiguous(total_k, Hkv, d),
                      contiguous(total_k, Hkv, d), contiguous(total_q, Hq, d), cu_seqlens_q, cu_seqlens_k, num_seqs,
                      total_q, total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, causal ? 1 : 0, dtype, stream,
                      !none && !causal, wl, wr);
}

fa_status fa_varlen_bwd_window(const void* q, const void* k, const void* v, const void* o, const float* lse,
                               const void* dout, void* dq, void* dk, void* dv, void* workspace,
                               const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs, int total_q,
                               int total_k, int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv, int d, float scale,
                               int window_left, int window_right, fa_dtype dtype, fa_stream_t stream) {
    const int wl = window_left < 0 ? -1 : window_left, wr = window_right < 0 ? -1 : window_right;
    const bool masked = wl >= 0 || wr >= 0;
    return varlen_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q,
                      total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, masked ? 1 : 0, dtype, stream, wl, wr);
}

fa_status fa_varlen_fwd_window_anchor(const void* q, const void* k, const void* v, void* o, float* lse,
                                      const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs, int total_q,
                                      int total_k, int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv, int d,
                                      float scale, int window_left, int window_right, int n_anchor, fa_dtype dtype,
                                      fa_stream_t stream) {
    if (n_anchor < 0) return FA_ERR_INVALID_ARG;
    const int wl = window_left < 0 ? -1 : window_left, wr = window_right < 0 ? -1 : window_right;
    if (n_anchor == 0 || wl < 0)  // no anchors, or nothing below the window to add
        return fa_varlen_fwd_window(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q, total_k,
                                    max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, wl, wr, dtype, stream);
    return fwd_varlen(q, k, v, o, lse, contiguous(total_q, Hq, d), contiguous(total_k, Hkv, d),
                      contiguous(total_k, Hkv, d), contiguous(total_q, Hq, d), cu_seqlens_q, cu_seqlens_k, num_seqs,
                      total_q, total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, 0, dtype, stream, true, wl, wr,
                      n_anchor);
}

fa_status fa_varlen_bwd_window_anchor(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                      const void* dout, void* dq, void* dk, void* dv, void* workspace,
                                      const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs, int total_q,
                                      int total_k, int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv, int d,
                                      float scale, int window_left, int window_right, int n_anchor, fa_dtype dtype,
                                      fa_stream_t stream) {
    if (n_anchor < 0) return FA_ERR_INVALID_ARG;
    const int wl = window_left < 0 ? -1 : window_left, wr = window_right < 0 ? -1 : window_right;
    const bool masked = wl >= 0 || wr >= 0;
    return varlen_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q,
                      total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, masked ? 1 : 0, dtype, stream, wl, wr,
                      wl >= 0 ? n_anchor : 0);
}

fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, const float* q_scale, const float* k_scale,
                     const float* v_scale, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                     float scale, int causal, fa_stream_t stream) {
    return fwd_fp8(q, k, v, q_scale, k_scale, v_scale, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream);
}

size_t fa_decode_workspace_size(int B, int Hq, int Hkv, int Nq, int d) {
    DecWs w;
    return dec_ws(B, Hq, Hkv, Nq, d, w) ? w.total : 0;
}

fa_status fa_decode(const void* q, const void* k, const void* v, void* o, float* lse, const int* cache_seqlens,
                    void* workspace, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                    fa_dtype dtype, fa_stream_t stream) {
    return decode_common(q, k, v, o, lse, cache_seqlens, nullptr, workspace, B, Hq, Hkv, Nq, Nk, false, 0, 0, 0, d,
                         scale, causal, dtype, stream);
}

fa_status fa_decode_paged(const void* q, const void* k_pages, const void* v_pages, void* o, float* lse,
                          const int* cache_seqlens, const int* block_table, void* workspace, int B, int Hq, int Hkv,
                          int Nq, int num_pages, int page_size, int max_pages, int d, float scale, int causal,
                          fa_dtype dtype, fa_stream_t stream) {
    return decode_common(q, k_pages, v_pages, o, lse, cache_seqlens, block_table, workspace, B, Hq, Hkv, Nq, 0, true,
                         num_pages, page_size, max_pages, d, scale, causal, dtype, stream);
}

fa_status fa_get_last_device_error(fa_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_fa_error, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    if (v == 0) return FA_OK;
    g_last_site = v;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_fa_error, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    if (v == fa::kErrSeqlenBound) return FA_ERR_INVALID_ARG;
    return (v >= fa::kErrTimeoutBase && v < fa::kErrSmemAlign) ? FA_ERR_TIMEOUT : FA_ERR_CUDA;
}

int fa_get_last_device_error_site(void) { return g_last_site; }

fa_status fa_selftest_bounded_wait(fa_stream_t stream) {
    int* err = error_word();
    if (!err) return FA_ERR_CUDA;
    fa_selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(err);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

void fa_bwd_set_timing_events(void* before, void* after) {
    g_bwd_ev_before = static_cast<cudaEvent_t>(before);
    g_bwd_ev_after = static_cast<cudaEvent_t>(after);
}

}  // extern "C"

