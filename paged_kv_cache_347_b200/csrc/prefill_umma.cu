// Causal multi-token attention over the paged cache on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory), sm_100a.
//
// Same quantity as prefill_tc.cu (mbrenndoerfer.com "Paged Attention >
// Summary", bullet 3; paweldubiel.com "PagedAttention", "Mechanism and
// details"): row r of a sequence's chunk, at position L - n + r, attends to
// positions 0..L-n+r through the block table.
//
// CTA = 128 (token, query head) rows: 128/G chunk tokens of one KV head g of
// one sequence; the context is walked in stages of 128 keys.  Eleven warps:
//   * warps 0-7, softmax: two threads per row -- warp w serves TMEM lanes
//     32 (w % 4) .. +31 (the rows) and keys 64 (w / 4) .. +63 of each stage.
//     Per stage a thread reads its 64 S values from TMEM, applies the causal
//     mask, agrees the row maximum with its partner thread (through shared
//     memory and an mbarrier), writes P = 2^(x - m) into TMEM as 16-bit
//     high part + remainder, and rescales its half of the O row when the
//     maximum has grown by more than 2^8; at the end it divides by the summed
//     weights and stores its half of the row;
//   * warps 8 and 9: TMA producers of the K and the V stages, gathered block
//     by block through the table into two rings: a K slot is free again as
//     soon as its S MMA has run, a V slot once its PV MMA has;
//   * warp 10, one thread: issues the UMMAs --
//       S[128 x 128]  = Q[128 x D] . K_stage^T       (Q, K from shared memory)
//       O[128 x D]   += P[128 x 128] . V_stage       (P from TMEM, V N-major)
//     and commits them to mbarriers.  S is double-buffered, so S of stage
//     i+1 runs on the tensor core while the softmax works on stage i.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O [256,256+D),
// P high part [384,448), P remainder [448,512).
//
// Every wait is bounded (~2 s); on a timeout the CTA records
// PA_DEVERR_TIMEOUT, the other warps stop waiting, the producer waits
// (bounded) for its copies, warp 0 waits for the MMAs and frees the TMEM.
#include <math.h>

#include <mutex>

#include "decode_common.cuh"
#include "umma.cuh"

namespace pa {
namespace pu {

constexpr int kM = 128;              // rows per CTA
constexpr int kKeys = 128;           // keys per stage
constexpr int kSoftmaxThreads = 256; // 8 warps, two threads per row
constexpr int kThreads = kSoftmaxThreads + 96;  // + K producer, V producer, MMA issuer
constexpr int kTmemCols = 512;
constexpr int kColO = 256, kColPHi = 384, kColPLo = 448;
constexpr int kRowBytes = 128;       // one 64-element piece of a 16-bit row

template <int D, int BS, int NK, int NV>
struct Cfg {
    static constexpr int kPieces = D / 64;
    static constexpr int kQPiece = kM * kRowBytes;        // 16 KB
    static constexpr int kQBytes = kPieces * kQPiece;
    static constexpr int kKVPiece = kKeys * kRowBytes;    // 16 KB
    static constexpr int kStageBytes = kPieces * kKVPiece;  // one K or V stage
    static constexpr int kQOffset = 0;
    static constexpr int kKOffset = kQBytes;                        // K ring [NK]
    static constexpr int kVOffset = kKOffset + NK * kStageBytes;    // V ring [NV]
    static constexpr int kXchOffset = kVOffset + NV * kStageBytes;  // float [2][2][128]
    static constexpr int kBarOffset = kXchOffset + 2 * 2 * kM * 4;
    // k_full[NK] k_empty[NK] v_full[NV] v_empty[NV] s_full[2] s_empty[2]
    // p_full pv_done q_full mma_done xchg[4]
    static constexpr int kNumBars = 2 * NK + 2 * NV + 4 + 4 + 4;
    static constexpr int kTmemSlot = kBarOffset + kNumBars * 8;
    static constexpr int kAbortOffset = kTmemSlot + 16;
    static constexpr int kSmemBytes = kAbortOffset + 16;
    static constexpr int kDynSmem = kSmemBytes + 1024;
    static constexpr int kBlocksPerStage = kKeys / BS;
    static_assert(kDynSmem <= 227 * 1024, "shared memory");
    static_assert(kKeys % BS == 0 && kBlocksPerStage <= 32, "block size");
    static_assert(D == 64 || D == 128, "head size");
};

// A bounded mbarrier wait taken by a whole warp, with one outcome for all
// its lanes (the tcgen05 loads and stores that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, abort_flag));
}

// Two weights -> their 16-bit high parts and remainders, one 32-bit word each
// (lower key in the low half).  bf16: the high part is the upper 16 bits of
// the fp32 pattern, the remainder x - hi is exact in fp32 and is rounded to
// its upper 16 bits; integer and permute instructions only.  f16 uses the
// hardware conversions.
template <typename T> struct PSplit;
template <> struct PSplit<__nv_bfloat16> {
    __device__ __forceinline__ static void run(float x0, float x1, uint32_t &hi, uint32_t &lo) {
        const uint32_t a = __float_as_uint(x0), b = __float_as_uint(x1);
        hi = __byte_perm(a, b, 0x7632);  // truncated: 0 <= x - hi < 2^-7 x
        const float r0 = x0 - __uint_as_float(a & 0xffff0000u);
        const float r1 = x1 - __uint_as_float(b & 0xffff0000u);
        // remainder rounded half up in magnitude: |x - hi - lo| <= 2^-16 x
        lo = __byte_perm(__float_as_uint(r0) + 0x8000u, __float_as_uint(r1) + 0x8000u, 0x7632);
    }
};
template <> struct PSplit<__half> {
    __device__ __forceinline__ static void run(float x0, float x1, uint32_t &hi, uint32_t &lo) {
        hi = Mma<__half>::pack(x0, x1);
        lo = Mma<__half>::pack(x0 - Mma<__half>::lo(hi), x1 - Mma<__half>::hi(hi));
    }
};

template <typename T, int D, int BS, int NK, int NV>
__global__ void __launch_bounds__(kThreads, 1) prefill_umma_kernel(
    const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
    const PrefillParams p) {
    using C = Cfg<D, BS, NK, NV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    pdl_wait_prior_grid();

    const int qt = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
    const int G = p.num_heads / p.num_kv_heads;
    const int TQ = p.tokens_per_cta;  // 128 / G
    const int q0 = __ldg(p.cu_q + s);
    const int n = __ldg(p.cu_q + s + 1) - q0;
    const int L = __ldg(p.seq_lens + s);
    if (n < 0 || n > L || L > p.max_seq_len || n > p.max_q_len ||
        (int64_t)(L + BS - 1) / BS > p.max_blocks_per_seq) {
        if (qt == 0 && g == 0 && threadIdx.x == 0) raise_device_error(p.err, PA_DEVERR_SEQLEN);
        return;
    }
    const int tok0 = qt * TQ;
    if (tok0 >= n) return;  // uniform, before any barrier or TMEM use
    const int ntok = min(TQ, n - tok0);
    const int pos0 = L - n + tok0;
    const int nkeys = pos0 + ntok;
    const int nstages = (nkeys + kKeys - 1) / kKeys;
    const int nblk = (nkeys + BS - 1) / BS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const uint32_t sbase = smem_u32(smem);
    const uint32_t q_s = sbase + C::kQOffset, k_s = sbase + C::kKOffset,
                   v_s = sbase + C::kVOffset;
    const uint32_t bar0 = sbase + C::kBarOffset;
    const uint32_t k_full = bar0, k_empty = k_full + 8 * NK, v_full = k_empty + 8 * NK,
                   v_empty = v_full + 8 * NV, s_full = v_empty + 8 * NV, s_empty = s_full + 16,
                   p_full = s_empty + 16, pv_done = p_full + 8, q_full = pv_done + 8,
                   mma_done = q_full + 8, xchg = mma_done + 8;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kAbortOffset);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + C::kTmemSlot);

    if (threadIdx.x == 0) {
        for (int i = 0; i < NK; ++i) {
            mbar_init(k_full + 8 * i, 1);
            mbar_init(k_empty + 8 * i, 1);
        }
        for (int i = 0; i < NV; ++i) {
            mbar_init(v_full + 8 * i, 1);
            mbar_init(v_empty + 8 * i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(s_full + 8 * i, 1);
            mbar_init(s_empty + 8 * i, kSoftmaxThreads);
        }
        mbar_init(p_full, kSoftmaxThreads);
        mbar_init(pv_done, 1);
        mbar_init(q_full, kSoftmaxThreads);
        mbar_init(mma_done, 1);
        for (int i = 0; i < 4; ++i) mbar_init(xchg + 8 * i, 64);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 0) {
        umma::tmem_alloc(sbase + C::kTmemSlot, kTmemCols);
        umma::tmem_relinquish();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    // ------------------------------------------------------------ producer
    // warp 8 loads the K stages, warp 9 the V stages, each at its own pace
    if (warp == 8 || warp == 9) {
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
        const uint64_t policy = l2_policy_evict_first();
        // lane j < jn(i) holds the physical block of the stage's j-th table entry
        auto lookup = [&](int i) -> int {
            const int jb = i * C::kBlocksPerStage;
            const int jn = min(C::kBlocksPerStage, nblk - jb);
            if (lane >= jn) return -1;
            const int b = checked_block_row(p.block_tables, p.max_blocks_per_seq, p.num_blocks,
                                            p.err, s, jb + lane);
            return b < 0 ? p.num_blocks : b;  // out of range: the copy reads the fill value
        };
        // one K or V stage: wait for the slot, announce the bytes, lane j copies block j
        auto load = [&](int i, int blk, const CUtensorMap *map, uint32_t ring, uint32_t full,
                        uint32_t empty, int nslots) -> bool {
            const int slot = i % nslots;
            int stop = 0;
            if (lane == 0 && i >= nslots &&
                !mbar_wait_bounded(empty + 8 * slot, ((i / nslots) - 1) & 1, abort_flag))
                stop = 1;
            if (__shfl_sync(0xffffffffu, stop, 0)) return false;
            const int jn = min(C::kBlocksPerStage, nblk - i * C::kBlocksPerStage);
            if (lane == 0) mbar_arrive_expect_tx(full + 8 * slot, (uint32_t)(jn * 2 * BS * D));
            __syncwarp();
            if (blk >= 0) {
                const uint32_t dst = ring + slot * C::kStageBytes + lane * BS * kRowBytes;
                const int y = (blk * p.num_kv_heads + g) * BS;
#pragma unroll
                for (int pc = 0; pc < C::kPieces; ++pc)
                    tma_load_2d(dst + pc * C::kKVPiece, map, pc * 64, y, full + 8 * slot, policy);
            }
            return true;
        };
        const bool is_k = warp == 8;
        const CUtensorMap *map = is_k ? &tmap_k : &tmap_v;
        const uint32_t ring = is_k ? k_s : v_s, full = is_k ? k_full : v_full,
                       empty = is_k ? k_empty : v_empty;
        const int nslots = is_k ? NK : NV;
        int issued = 0;
        for (int i = 0; i < nstages; ++i) {
            if (!load(i, lookup(i), map, ring, full, empty, nslots)) break;
            issued = i + 1;
        }
        if (lane == 0) {
            if (issued < nstages) {
                raise_device_error(p.err, PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            // wait (bounded) for the copies still in flight
            for (int i = max(0, issued - nslots); i < issued; ++i)
                mbar_wait_bounded(full + 8 * (i % nslots), (i / nslots) & 1, nullptr);
        }
        return;
    }

    // ------------------------------------------------------------ MMA issuer
    if (warp == 10) {
        if (lane == 0) {
            constexpr uint32_t fmt = StoreT<T>::kCode == PA_BF16 ? 1u : 0u;
            constexpr uint32_t idesc_s = umma::idesc_f16(fmt, kM, kKeys, 0);
            constexpr uint32_t idesc_o = umma::idesc_f16(fmt, kM, D, 1);
            bool ok = mbar_wait_bounded(q_full, 0, abort_flag);
            // S_i = Q . K_i^T into TMEM columns 128 * (i % 2)
            auto issue_s = [&](int i) -> bool {
                const int buf = i % NK;
                if (!mbar_wait_bounded(k_full + 8 * buf, (i / NK) & 1, abort_flag)) return false;
                if (i >= 2 && !mbar_wait_bounded(s_empty + 8 * (i % 2), ((i / 2) - 1) & 1,
                                                 abort_flag))
                    return false;
                umma::fence_after_sync();
                const uint32_t kst = k_s + buf * C::kStageBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t a = umma::smem_desc_sw128(
                        q_s + (kk >> 2) * C::kQPiece + (kk & 3) * 32, 16, 1024);
                    const uint64_t b = umma::smem_desc_sw128(
                        kst + (kk >> 2) * C::kKVPiece + (kk & 3) * 32, 16, 1024);
                    umma::mma_f16(tmem + (i % 2) * kKeys, a, b, idesc_s, kk > 0);
                }
                umma::commit(s_full + 8 * (i % 2));
                umma::commit(k_empty + 8 * buf);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int i = 0; ok && i < nstages; ++i) {
                if (i + 1 < nstages && !issue_s(i + 1)) {
                    ok = false;
                    break;
                }
                // O += P_i . V_i once the softmax has written P_i
                if (!mbar_wait_bounded(p_full, i & 1, abort_flag) ||
                    !mbar_wait_bounded(v_full + 8 * (i % NV), (i / NV) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                umma::fence_after_sync();
                const uint32_t vst = v_s + (i % NV) * C::kStageBytes;
#pragma unroll
                for (int j = 0; j < kKeys / 16; ++j) {
                    // keys 16j..16j+15: V rows (8-row groups 1 KB apart), 64-column pieces 16 KB apart
                    const uint64_t b = umma::smem_desc_sw128(vst + j * 16 * kRowBytes,
                                                             C::kKVPiece, 1024);
                    umma::mma_f16_ts(tmem + kColO, tmem + kColPHi + 8 * j, b, idesc_o,
                                     (i > 0 || j > 0) ? 1u : 0u);
                    umma::mma_f16_ts(tmem + kColO, tmem + kColPLo + 8 * j, b, idesc_o, 1u);
                }
                umma::commit(pv_done);
                umma::commit(v_empty + 8 * (i % NV));
            }
            if (!ok) {
                raise_device_error(p.err, PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            umma::commit(mma_done);  // arrives when every MMA issued above is done
        }
        return;
    }

    // ------------------------------------------------------------ softmax warps
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;  // row == TMEM lane
    const int t = r / G, hh = r - t * G;
    const bool valid = t < ntok && r < TQ * G;
    const int qp = valid ? pos0 + t : nkeys - 1;
    const int64_t qrow = ((int64_t)(q0 + tok0 + t) * p.num_heads + g * G + hh) * D;
    // S is computed with sign(scale) folded into Q (a sign-bit flip, exact),
    // so that the logit scale applied below is non-negative
    const uint32_t qflip = p.scale_log2 < 0.f ? 0x80008000u : 0u;
    const float sl2 = fabsf(p.scale_log2);
    {
        // this thread's half of the Q row -> swizzled K-major tile
        // (row r, 16-byte chunk c at c ^ (r & 7) within its 128-byte piece row)
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const T *>(p.q) + qrow);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
            const int c = half * (D / 16) + k;
            uint4 v = valid ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
            v.x ^= qflip; v.y ^= qflip; v.z ^= qflip; v.w ^= qflip;
            *reinterpret_cast<uint4 *>(smem + C::kQOffset + (c >> 3) * C::kQPiece +
                                       r * kRowBytes + (((c & 7) ^ (r & 7)) << 4)) = v;
        }
        umma::fence_proxy_async_smem();
        mbar_arrive(q_full);
    }
    float *xch = reinterpret_cast<float *>(smem + C::kXchOffset);  // [parity][half][row]
    const uint32_t my_xchg = xchg + 8 * quarter;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < nstages; ++i) {
        const int sb = i & 1;
        if (!warp_wait(s_full + 8 * sb, (i >> 1) & 1, abort_flag)) {
            ok = false;
            break;
        }
        umma::fence_after_sync();
        uint32_t sr[2][32];
        umma::ld32(lane_base + sb * kKeys + half * 64, sr[0]);
        umma::ld32(lane_base + sb * kKeys + half * 64 + 32, sr[1]);
        umma::wait_ld();
        umma::fence_before_sync();
        mbar_arrive(s_empty + 8 * sb);
        const int kb = i * kKeys + half * 64;
        float sv[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) sv[c] = __uint_as_float(sr[c >> 5][c & 31]);
        // Keys past a row's position exist only on stages reaching beyond the
        // first chunk token's position (the test is uniform over the CTA);
        // there the logits are scaled and masked here, elsewhere the scale is
        // applied inside the exponent's FMA.
        const bool masked = i * kKeys + kKeys - 1 > pos0;
        float mx;
        {
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (masked) {
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    sv[c] = kb + c > qp ? -INFINITY : sv[c] * sl2;
                    m4[c & 3] = fmaxf(m4[c & 3], sv[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c) m4[c & 3] = fmaxf(m4[c & 3], sv[c]);
            }
            mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            if (!masked) mx *= sl2;  // sl2 >= 0
        }
        // the row maximum of this stage over both halves
        xch[(sb * 2 + half) * kM + r] = mx;
        mbar_arrive(my_xchg);
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(my_xchg, i & 1, abort_flag))) {
            ok = false;
            break;
        }
        mx = fmaxf(mx, xch[(sb * 2 + (half ^ 1)) * kM + r]);
        // the running max moves only when it grows by more than 8 (log2 units):
        // weights then stay below 2^8 and O is rescaled rarely
        float alpha = 1.f;
        bool rescale = false;
        if (mx > m + 8.f) {
            alpha = umma::ex2(m - mx);  // 0 on the first stage (m = -inf)
            rescale = m != -INFINITY;
            m = mx;
        }
        // weights 2^(x - m), summed and split into TMEM words as they are made
        const float fm = masked ? 1.f : sl2;
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t ph[32], pl[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const float p0 = umma::ex2(fmaf(sv[2 * e], fm, -m));
            const float p1 = umma::ex2(fmaf(sv[2 * e + 1], fm, -m));
            s4[e & 3] += p0 + p1;
            PSplit<T>::run(p0, p1, ph[e], pl[e]);
        }
        l = l * alpha + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
        // PV of stage i-1 must be done before O is rescaled and P overwritten
        if (i > 0 && !warp_wait(pv_done, (i - 1) & 1, abort_flag)) {
            ok = false;
            break;
        }
        umma::fence_after_sync();
        umma::st32(lane_base + kColPHi + half * 32, ph);
        umma::st32(lane_base + kColPLo + half * 32, pl);
        if (__any_sync(0xffffffffu, rescale)) {  // warp-collective TMEM access
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
                uint32_t o[32];
                const uint32_t col = lane_base + kColO + half * (D / 2) + cb * 32;
                umma::ld32(col, o);
                umma::wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                umma::st32(col, o);
            }
        }
        if (i * kKeys + kKeys > nkeys) {
            // last stage: rows past the last key hold stale or unwritten data;
            // zero them in V so that their zero weights give exact zeros.  The
            // wait only orders these stores after the stage's copies.
            if (!warp_wait(v_full + 8 * (i % NV), (i / NV) & 1, abort_flag)) {
                ok = false;
                break;
            }
            const int first = nkeys - i * kKeys;  // rows [first, 128)
            uint8_t *vst = smem + C::kVOffset + (i % NV) * C::kStageBytes;
            for (int idx = threadIdx.x; idx < (kKeys - first) * C::kPieces * 8;
                 idx += kSoftmaxThreads) {
                const int row = first + idx / (C::kPieces * 8);
                const int rem = idx % (C::kPieces * 8);
                *reinterpret_cast<uint4 *>(vst + (rem >> 3) * C::kKVPiece + row * kRowBytes +
                                           ((rem & 7) << 4)) = make_uint4(0u, 0u, 0u, 0u);
            }
            umma::fence_proxy_async_smem();
        }
        umma::wait_st();
        umma::fence_before_sync();
        mbar_arrive(p_full);
    }
    if (ok && !warp_wait(pv_done, (nstages - 1) & 1, abort_flag)) ok = false;
    if (ok) {
        // the two halves' weight sums
        xch[((nstages & 1) * 2 + half) * kM + r] = l;
        mbar_arrive(my_xchg);
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(my_xchg, nstages & 1, abort_flag));
    }
    if (ok) {
        l += xch[((nstages & 1) * 2 + (half ^ 1)) * kM + r];
        umma::fence_after_sync();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float *dst = p.out + qrow + half * (D / 2);
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb) {
            uint32_t o[32];
            umma::ld32(lane_base + kColO + half * (D / 2) + cb * 32, o);
            umma::wait_ld();
            if (valid) {
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(dst + cb * 32 + e) =
                        make_float4(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv,
                                    __uint_as_float(o[e + 2]) * inv,
                                    __uint_as_float(o[e + 3]) * inv);
            }
        }
    } else if (lane == 0) {
        raise_device_error(p.err, PA_DEVERR_TIMEOUT);
        *abort_flag = 1;  // the other warps stop waiting
    }
    // TMEM is freed once every MMA of this CTA has completed and every
    // softmax warp is done with it
    umma::fence_before_sync();
    named_barrier_sync(1, kSoftmaxThreads);
    if (warp == 0) {
        mbar_wait_bounded(mma_done, 0, nullptr);
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, kTmemCols);
    }
    pdl_launch_dependents();
}

template <typename T, int D, int BS>
static cudaError_t launch_inst(const PrefillParams &p, const CUtensorMap &mk,
                               const CUtensorMap &mv, cudaStream_t stream) {
    constexpr int NK = D == 128 ? 3 : 4, NV = D == 128 ? 2 : 4;
    using C = Cfg<D, BS, NK, NV>;
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(prefill_umma_kernel<T, D, BS, NK, NV>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kDynSmem);
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((p.max_q_len + p.tokens_per_cta - 1) / p.tokens_per_cta, p.num_kv_heads,
                       p.num_seqs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kDynSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_umma_kernel<T, D, BS, NK, NV>, mk, mv, p);
}

template <typename T, int D>
static cudaError_t launch_d(const PrefillParams &p, const CUtensorMap &mk, const CUtensorMap &mv,
                            cudaStream_t stream) {
    switch (p.block_size) {
    case 8: return launch_inst<T, D, 8>(p, mk, mv, stream);
    case 16: return launch_inst<T, D, 16>(p, mk, mv, stream);
    case 32: return launch_inst<T, D, 32>(p, mk, mv, stream);
    case 64: return launch_inst<T, D, 64>(p, mk, mv, stream);
    default: return cudaErrorNotSupported;
    }
}

}  // namespace pu

cudaError_t launch_prefill_umma(const PrefillParams &p, int dtype, cudaStream_t stream) {
    if (p.num_seqs == 0 || p.max_q_len == 0) return cudaSuccess;
    const int64_t rows = (int64_t)p.num_blocks * p.num_kv_heads * p.block_size;
    CUtensorMap mk, mv;
    if (!make_cache_tensor_map(&mk, p.k_cache, dtype, p.head_dim, rows, p.block_size) ||
        !make_cache_tensor_map(&mv, p.v_cache, dtype, p.head_dim, rows, p.block_size))
        return cudaErrorInvalidValue;
    if (dtype == PA_BF16)
        return p.head_dim == 128 ? pu::launch_d<__nv_bfloat16, 128>(p, mk, mv, stream)
                                 : pu::launch_d<__nv_bfloat16, 64>(p, mk, mv, stream);
    return p.head_dim == 128 ? pu::launch_d<__half, 128>(p, mk, mv, stream)
                             : pu::launch_d<__half, 64>(p, mk, mv, stream);
}

}  // namespace pa
