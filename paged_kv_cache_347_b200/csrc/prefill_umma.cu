// Causal multi-token attention over the paged cache on the 5th-generation
// tensor cores (tcgen05, operands and accumulators in tensor memory), sm_100a.
//
// Same quantity as prefill_tc.cu (mbrenndoerfer.com "Paged Attention >
// Summary", bullet 3; paweldubiel.com "PagedAttention", "Mechanism and
// details"): row r of a sequence's chunk, at position L - n + r, attends to
// positions 0..L-n+r through the block table.
//
// Tile = 128 (token, query head) rows: 128/G chunk tokens of one KV head g of
// one sequence, walking the context in stages of 128 keys.  A CTA takes one
// tile, or (the persistent form) one CTA per SM walks every gridDim-th tile,
// with stage and tile counters running on across tiles.  Twelve warps:
//   * warps 0-7, softmax: warp w serves TMEM lanes 32 (w % 4) .. +31 (the
//     rows) and keys 64 (w / 4) .. +63 of each stage, so each row has two
//     threads, which agree its maximum through shared memory.  A thread reads
//     its 64 S values from TMEM, writes P = 2^(x - m) as 16-bit high part +
//     remainder into the same TMEM columns, and rescales its half of the O
//     row when the maximum has grown by more than 2^8; at the end the halves'
//     weight sums are added and each thread divides and stores its half row;
//   * warps 8 and 9: TMA producers of the K and the V stages, gathered block
//     by block through the table into two rings;
//   * warps 10 and 11, one thread each, issue the UMMAs:
//       S(i)  [128 x 128] = Q . K_i^T      (Q from TMEM, K from shared memory)
//       PV(i) O [128 x D] += P_i . V_i      (P from TMEM, V N-major, twice:
//                                            high part and remainder)
//     S is double-buffered, so the softmax of stage i+1 can start as soon as
//     it ends stage i; S(i+2), which overwrites the columns PV(i) reads, is
//     issued once PV(i) has completed.
// Between two tiles the softmax warps put the next tile's Q into the other Q
// buffer as soon as the tile's last PV is done (the S thread can start the
// next tile), read O out of TMEM and count it on o_free (the next tile's
// first PV starts O afresh), then normalise and store the rows.
// TMEM (512 columns): S/P buffers [0,128) and [128,256), O [256,256+D),
// two Q buffers [384,384+D/2) and [384+D/2,384+D).  In P, key block j (keys
// 16j..16j+15) holds its high parts in columns 16j..16j+7 and its remainders
// in 16j+8..16j+15, two keys per column; Q holds two elements of a row per
// column.
//
// The one-fp16-P form (kP16, one tile per CTA): each weight is rounded once
// to fp16, and P takes 64 columns of its own, [448, 512) (free with a single
// Q buffer; key block j at 448 + 8 j, a thread's 64 keys in 32 of them), so
// S(i+2) waits only until the softmax has read S(i), and the softmax waits
// for PV(i-1) to have read P(i-1) before it writes P(i).  PV(i) is one MMA
// per key block with P and V both f16.  Against a bf16 cache a fourth
// warpgroup (warps 12-15) rewrites each landed V stage in place as fp16
// (and zeroes the rows past the tile's last key) before the PV thread may
// read it; a V value beyond the fp16 range turns infinite there, which the
// epilogue finds in the output and reports as PA_DEVERR_RANGE.
//
// Every wait is bounded (~2 s); on a timeout the CTA records
// PA_DEVERR_TIMEOUT, the other warps stop waiting, the producers wait
// (bounded) for their copies, warp 0 waits for the MMAs and frees the TMEM.
#include <math.h>

#include <algorithm>
#include <climits>
#include <mutex>
#include <type_traits>

#include "decode_common.cuh"
#include "prefill_common.cuh"
#include "umma.cuh"

namespace pa {
namespace pu {

constexpr int kM = 128;               // rows per CTA
constexpr int kKeys = 128;            // keys per stage
constexpr int kSoftmaxThreads = 256;  // 8 warps, two threads per row
constexpr int kThreads = kSoftmaxThreads + 128;  // + K, V producers, S, PV issuers
// + one warpgroup converting the V stages of a bf16 cache to fp16 (one-fp16-P form)
constexpr int kConvThreads = 128;
__host__ __device__ constexpr int threads_for(bool conv) {
    return conv ? kThreads + kConvThreads : kThreads;
}
constexpr int kTmemCols = 512;
constexpr int kColO = 256, kColQ = 384;
// the one-fp16-P form (one tile per CTA, so one Q buffer): P in columns of
// its own, [448, 512), key block j at kColP + 8 j
constexpr int kColP = 448;
constexpr int kRowBytes = 128;        // one 64-element piece of a 16-bit row

template <int D, int BS, int NK, int NV>
struct Cfg {
    static constexpr int kPieces = D / 64;
    static constexpr int kKVPiece = kKeys * kRowBytes;      // 16 KB
    static constexpr int kStageBytes = kPieces * kKVPiece;  // one K or V stage
    static constexpr int kKOffset = 0;                              // K ring [NK]
    static constexpr int kVOffset = kKOffset + NK * kStageBytes;    // V ring [NV]
    static constexpr int kXchOffset = kVOffset + NV * kStageBytes;  // float [2][2][128]
    static constexpr int kBarOffset = kXchOffset + 2 * 2 * kM * 4;
    // k_full[NK] k_empty[NK] v_full[NV] v_empty[NV] s_full[2] p_full[2] pv_done[2]
    // q_full[2] o_free mma_done xchg[4] v_conv[NV]
    static constexpr int kNumBars = 2 * NK + 3 * NV + 6 + 4 + 4;
    static constexpr int kTmemSlot = kBarOffset + kNumBars * 8;
    static constexpr int kAbortOffset = kTmemSlot + 16;
    static constexpr int kSmemBytes = kAbortOffset + 16;
    static constexpr int kDynSmem = kSmemBytes + 1024;
    static constexpr int kBlocksPerStage = kKeys / BS;
    static_assert(kDynSmem <= 227 * 1024, "shared memory");
    static_assert(kKeys % BS == 0 && kBlocksPerStage <= 32, "block size");
    static_assert(D == 64 || D == 128, "head size");
    static_assert(kColO + D <= kColQ && kColQ + D <= kTmemCols, "tensor memory: two Q buffers");
};

// A bounded mbarrier wait taken by a whole warp, with one outcome for all
// its lanes (the tcgen05 loads and stores that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, abort_flag));
}

// Paired fp32 arithmetic (sm_100 f32x2 instructions): two lanes per instruction.
__device__ __forceinline__ uint64_t pk(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk(uint64_t r, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// max of three (sm_100 three-input max)
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Two weights -> their 16-bit high parts and remainders, one 32-bit word each
// (lower key in the low half).  bf16: the high part is the upper 16 bits of
// the fp32 pattern, the remainder x - hi is exact in fp32 and is cut to its
// upper 16 bits as well (one logic op, one add and one permute per weight);
// f16 uses the hardware conversions.
template <typename T> struct PSplit;
template <> struct PSplit<__nv_bfloat16> {
    __device__ __forceinline__ static void run(float x0, float x1, uint32_t &hi, uint32_t &lo) {
        const uint32_t a = __float_as_uint(x0), b = __float_as_uint(x1);
        hi = __byte_perm(a, b, 0x7632);  // truncated: 0 <= x - hi < 2^-7 x
        const float r0 = x0 - __uint_as_float(a & 0xffff0000u);
        const float r1 = x1 - __uint_as_float(b & 0xffff0000u);
        // remainder truncated too: 0 <= x - hi - lo < 2^-14 x
        lo = __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632);
    }
};
template <> struct PSplit<__half> {
    __device__ __forceinline__ static void run(float x0, float x1, uint32_t &hi, uint32_t &lo) {
        hi = Mma<__half>::pack(x0, x1);
        lo = Mma<__half>::pack(x0 - Mma<__half>::lo(hi), x1 - Mma<__half>::hi(hi));
    }
};

// Two bf16 values (one 32-bit word, the lower element in the low half) as
// two fp16 values in the same places: each widened to fp32 (exact), then
// rounded to the nearest fp16.  Exact for magnitudes in [2^-14, 65504];
// smaller ones keep 2^-24 absolute precision, 65536 and above become
// infinite.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
    return Mma<__half>::pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// What a CTA needs of one token tile: its sequence and KV head, where its
// rows start, how many keys it attends to.
struct Tile {
    int s, g, q0, tok0, ntok, pos0, nkeys, nstages, nblk;
};

// Tile u of the launch.  One tile per CTA: the 3-D grid, token tiles that
// attend to the most keys first within a (sequence, KV head).  Persistent:
// the same order as a list (sequence, then KV head, then token tile, longest
// first), CTA c taking tiles c, c + gridDim.x, ...: the CTAs at work at any
// time hold the tiles of a few (sequence, KV head) pairs, which share their
// K/V through L2, and each CTA's tiles mix long and short ones.  Every role
// of the CTA calls
// this with the same u and gets the same answer; false: nothing to do
// (an empty tile, or a sequence whose lengths break the bounds, which
// `report` records).
template <int BS, bool kPersist>
__device__ __forceinline__ bool describe_tile(const PrefillParams &p, int u, bool report,
                                              Tile &t) {
    const int TQ = p.tokens_per_cta;
    const int X = (p.max_q_len + TQ - 1) / TQ;  // token tiles per (sequence, KV head)
    int qt, g, s;
    if constexpr (kPersist) {
        qt = X - 1 - u % X;
        g = (u / X) % p.num_kv_heads;
        s = u / (X * p.num_kv_heads);
    } else {
        qt = gridDim.x - 1 - blockIdx.x;
        g = blockIdx.y;
        s = blockIdx.z;
    }
    const int q0 = __ldg(p.cu_q + s);
    const int n = __ldg(p.cu_q + s + 1) - q0;
    const int L = __ldg(p.seq_lens + s);
    if (n < 0 || n > L || L > p.max_seq_len || n > p.max_q_len ||
        (int64_t)(L + BS - 1) / BS > p.max_blocks_per_seq) {
        if (report && qt == 0 && g == 0) raise_device_error(p.err, PA_DEVERR_SEQLEN);
        return false;
    }
    const int tok0 = qt * TQ;
    if (tok0 >= n) return false;
    t.s = s;
    t.g = g;
    t.q0 = q0;
    t.tok0 = tok0;
    t.ntok = min(TQ, n - tok0);
    t.pos0 = L - n + tok0;
    t.nkeys = t.pos0 + t.ntok;
    t.nstages = (t.nkeys + kKeys - 1) / kKeys;
    t.nblk = (t.nkeys + BS - 1) / BS;
    return true;
}

template <typename T, int D, int BS, int NK, int NV, bool kPersist, bool kP16>
__global__ void __launch_bounds__(threads_for(kP16 && std::is_same<T, __nv_bfloat16>::value), 1)
    prefill_umma_kernel(const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v, const PrefillParams p) {
    using C = Cfg<D, BS, NK, NV>;
    // one fp16 P against a bf16 cache: V converted to fp16 in shared memory
    constexpr bool kConv = kP16 && std::is_same<T, __nv_bfloat16>::value;
    static_assert(!(kP16 && kPersist), "the one-fp16-P form takes one tile per CTA");
    static_assert(!kP16 || (kColQ + D / 2 <= kColP && kColP + kKeys / 2 <= kTmemCols),
                  "tensor memory: P columns beside the one Q buffer");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    pdl_wait_prior_grid();

    const int G = p.num_heads / p.num_kv_heads;
    const int TQ = p.tokens_per_cta;  // 128 / G
    const int ntiles =
        kPersist ? ((p.max_q_len + TQ - 1) / TQ) * p.num_kv_heads * p.num_seqs : 1;
    const int u0 = kPersist ? (int)blockIdx.x : 0;
    const int ustep = kPersist ? (int)gridDim.x : 1;
    if constexpr (!kPersist) {
        Tile t;
        // uniform over the CTA, before any barrier or TMEM use
        if (!describe_tile<BS, false>(p, 0, threadIdx.x == 0, t)) return;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const uint32_t sbase = smem_u32(smem);
    const uint32_t k_s = sbase + C::kKOffset, v_s = sbase + C::kVOffset;
    const uint32_t bar0 = sbase + C::kBarOffset;
    const uint32_t k_full = bar0, k_empty = k_full + 8 * NK, v_full = k_empty + 8 * NK,
                   v_empty = v_full + 8 * NV, s_full = v_empty + 8 * NV, p_full = s_full + 16,
                   pv_done = p_full + 16, q_full = pv_done + 16, o_free = q_full + 16,
                   mma_done = o_free + 8, xchg = mma_done + 8, v_conv = xchg + 32;
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
        // s_full, p_full and pv_done once per S buffer, q_full once per Q
        // buffer: a phase is never waited on two completions behind
        for (int b = 0; b < 2; ++b) {
            mbar_init(s_full + 8 * b, 1);
            mbar_init(p_full + 8 * b, kSoftmaxThreads);
            mbar_init(pv_done + 8 * b, 1);
            mbar_init(q_full + 8 * b, kSoftmaxThreads);
        }
        mbar_init(o_free, kSoftmaxThreads);  // a tile's O read out of TMEM
        mbar_init(mma_done, 2);              // both issuing threads
        for (int q = 0; q < 4; ++q) mbar_init(xchg + 8 * q, 64);
        for (int i = 0; i < NV; ++i) mbar_init(v_conv + 8 * i, kConvThreads);
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

    // ------------------------------------------------------------ producers
    // warp 8 loads the K stages, warp 9 the V stages, each at its own pace;
    // the ring runs on across the CTA's tiles (gi counts stages over all of
    // them)
    if (warp == 8 || warp == 9) {
        const bool is_k = warp == 8;
        const CUtensorMap *map = is_k ? &tmap_k : &tmap_v;
        if (lane == 0) prefetch_tensormap(map);
        const uint64_t policy = l2_policy_evict_normal();
        const uint32_t ring = is_k ? k_s : v_s, full = is_k ? k_full : v_full,
                       empty = is_k ? k_empty : v_empty;
        const int nslots = is_k ? NK : NV;
        int gi = 0;  // stages issued
        bool stop = false;
        for (int u = u0; !stop && u < ntiles; u += ustep) {
            Tile t;
            if (!describe_tile<BS, kPersist>(p, u, false, t)) continue;
            for (int i = 0; i < t.nstages; ++i) {
                const int slot = gi % nslots;
                const int jb = i * C::kBlocksPerStage;
                const int jn = min(C::kBlocksPerStage, t.nblk - jb);
                // lane j < jn holds the physical block of the stage's j-th table entry
                int blk = -1;
                if (lane < jn) {
                    const int b = checked_block_row(p.block_tables, p.max_blocks_per_seq,
                                                    p.num_blocks, p.err, t.s, jb + lane);
                    blk = b < 0 ? p.num_blocks : b;  // out of range: the copy reads the fill value
                }
                int quit = 0;
                if (lane == 0 && gi >= nslots &&
                    !mbar_wait_bounded(empty + 8 * slot, ((gi / nslots) - 1) & 1, abort_flag))
                    quit = 1;
                if (__shfl_sync(0xffffffffu, quit, 0)) {
                    stop = true;
                    break;
                }
                if (lane == 0) mbar_arrive_expect_tx(full + 8 * slot, (uint32_t)(jn * 2 * BS * D));
                __syncwarp();
                if (blk >= 0) {
                    const uint32_t dst = ring + slot * C::kStageBytes + lane * BS * kRowBytes;
                    const int y = (blk * p.num_kv_heads + t.g) * BS;
#pragma unroll
                    for (int pc = 0; pc < C::kPieces; ++pc)
                        tma_load_2d(dst + pc * C::kKVPiece, map, pc * 64, y, full + 8 * slot,
                                    policy);
                }
                ++gi;
            }
        }
        if (lane == 0) {
            if (stop) {
                raise_device_error(p.err, PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            // wait (bounded) for the copies still in flight
            for (int i = max(0, gi - nslots); i < gi; ++i)
                mbar_wait_bounded(full + 8 * (i % nslots), (i / nslots) & 1, nullptr);
        }
        return;
    }

    // ------------------------------------------------------------ V converters
    // (bf16 cache, one-fp16-P form) warps 12-15, one per SM sub-partition:
    // each V stage, once landed, is rewritten in place as fp16 (the 128-byte
    // swizzle moves 16-byte chunks within a row only, so a chunk converts
    // where it lies), rows past the tile's last key as zeros, and counted on
    // v_conv before the PV MMA reads it.
    if constexpr (kConv) {
        if (warp >= 12) {
            const int ct = threadIdx.x - kThreads;  // 0..127
            constexpr int kChunks = C::kPieces * kKeys * 8;  // 16-byte chunks per V stage
            static_assert(kChunks % kConvThreads == 0 && C::kKVPiece == kKeys * 8 * 16,
                          "V stage: whole chunks per converter thread, contiguous pieces");
            int gi = 0;
            bool ok = true;
            for (int u = u0; ok && u < ntiles; u += ustep) {
                Tile t;
                if (!describe_tile<BS, kPersist>(p, u, false, t)) continue;
                for (int i = 0; i < t.nstages; ++i, ++gi) {
                    const int slot = gi % NV;
                    if (!warp_wait(v_full + 8 * slot, (gi / NV) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int first = min(kKeys, t.nkeys - i * kKeys);  // rows >= first: zeros
                    // the stage's pieces are contiguous: chunk idx lies idx * 16 bytes
                    // in, in row (idx % 1024) / 8 of its piece
                    uint4 *a = reinterpret_cast<uint4 *>(smem + C::kVOffset +
                                                         slot * C::kStageBytes) + ct;
                    constexpr int kPer = kChunks / kConvThreads;
                    if (first == kKeys) {
                        uint4 w[kPer];
#pragma unroll
                        for (int k = 0; k < kPer; ++k) w[k] = a[k * kConvThreads];
#pragma unroll
                        for (int k = 0; k < kPer; ++k) {
                            w[k].x = bf16x2_to_f16x2(w[k].x);
                            w[k].y = bf16x2_to_f16x2(w[k].y);
                            w[k].z = bf16x2_to_f16x2(w[k].z);
                            w[k].w = bf16x2_to_f16x2(w[k].w);
                            a[k * kConvThreads] = w[k];
                        }
                    } else {
#pragma unroll 4
                        for (int k = 0; k < kPer; ++k) {
                            const int row = ((ct + k * kConvThreads) & (kKeys * 8 - 1)) >> 3;
                            uint4 w = make_uint4(0u, 0u, 0u, 0u);
                            if (row < first) {
                                w = a[k * kConvThreads];
                                w.x = bf16x2_to_f16x2(w.x);
                                w.y = bf16x2_to_f16x2(w.y);
                                w.z = bf16x2_to_f16x2(w.z);
                                w.w = bf16x2_to_f16x2(w.w);
                            }
                            a[k * kConvThreads] = w;
                        }
                    }
                    umma::fence_proxy_async_smem();  // visible to the tensor core's reads
                    mbar_arrive(v_conv + 8 * slot);
                }
            }
            if (!ok && lane == 0) {
                raise_device_error(p.err, PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            return;
        }
    }

    // ------------------------------------------------------------ MMA issuers
    // Warp 10 issues the S MMAs, warp 11 the PV MMAs, each from one thread, so
    // that neither waits behind the other's barrier checks.  MMAs of two
    // threads are not ordered against each other: S(i+2) overwrites the TMEM
    // columns PV(i) reads, so the S thread waits for PV(i) to complete.  Stage
    // indices (gi) and tile indices (tp) run on across the CTA's tiles: a
    // tile's Q sits in TMEM buffer tp % 2, and its first PV, which starts O
    // afresh, waits until the softmax warps have read out the previous tile's O.
    if (warp == 10 || warp == 11) {
        if (lane == 0) {
            constexpr uint32_t fmt = StoreT<T>::kCode == PA_BF16 ? 1u : 0u;
            bool ok = true;
            int gi = 0, tp = 0;
            for (int u = u0; ok && u < ntiles; u += ustep) {
                Tile t;
                if (!describe_tile<BS, kPersist>(p, u, false, t)) continue;
                if (warp == 10) {
                    constexpr uint32_t idesc_s = umma::idesc_f16(fmt, kM, kKeys, 0);
                    ok = mbar_wait_bounded(q_full + 8 * (tp & 1), (tp >> 1) & 1, abort_flag);
                    umma::fence_after_sync();
                    const uint32_t qcol = tmem + kColQ + (tp & 1) * (D / 2);
#pragma unroll 1
                    for (int i = 0; ok && i < t.nstages; ++i, ++gi) {
                        // S(gi) = Q . K^T into S buffer gi % 2, once PV(gi-2) has read it
                        const int slot = gi % NK;
                        // (with P in columns of its own, once the softmax has read
                        // S(gi-2): it arrives on p_full after that)
                        if (gi >= 2 && !mbar_wait_bounded((kP16 ? p_full : pv_done) + 8 * (gi & 1),
                                                          ((gi >> 1) - 1) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        if (!mbar_wait_bounded(k_full + 8 * slot, (gi / NK) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        umma::fence_after_sync();
                        // K rows: 8-row groups 1 KB apart; descriptors advance by (bytes >> 4)
                        const uint64_t b0 =
                            umma::smem_desc_sw128(k_s + slot * C::kStageBytes, 16, 1024);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t ka = ((kk >> 2) * C::kKVPiece + (kk & 3) * 32) >> 4;
                            umma::mma_f16_ts(tmem + (gi & 1) * kKeys, qcol + 8 * kk, b0 + ka,
                                             idesc_s, kk > 0);
                        }
                        umma::commit(s_full + 8 * (gi & 1));
                        umma::commit(k_empty + 8 * slot);
                    }
                } else {
                    // P as one fp16 per weight: P and V both f16
                    constexpr uint32_t idesc_o = umma::idesc_f16(kP16 ? 0u : fmt, kM, D, 1);
#pragma unroll 1
                    for (int i = 0; ok && i < t.nstages; ++i, ++gi) {
                        // O += P(gi) . V(gi) once the softmax has written P(gi)
                        const int slot = gi % NV;
                        // a bf16 V stage is read once the converters are done with it
                        const uint32_t v_ready = kConv ? v_conv : v_full;
                        if (!mbar_wait_bounded(p_full + 8 * (gi & 1), (gi >> 1) & 1, abort_flag) ||
                            !mbar_wait_bounded(v_ready + 8 * slot, (gi / NV) & 1, abort_flag) ||
                            (i == 0 && tp > 0 &&
                             !mbar_wait_bounded(o_free, (tp - 1) & 1, abort_flag))) {
                            ok = false;
                            break;
                        }
                        umma::fence_after_sync();
                        // V rows: 8-row groups 1 KB apart, 64-column pieces 16 KB apart
                        const uint64_t b0 = umma::smem_desc_sw128(v_s + slot * C::kStageBytes,
                                                                  C::kKVPiece, 1024);
                        [[maybe_unused]] const uint32_t pb = tmem + (gi & 1) * kKeys;
#pragma unroll
                        for (int j = 0; j < kKeys / 16; ++j) {  // keys 16j..16j+15
                            const uint64_t b = b0 + ((j * 16 * kRowBytes) >> 4);
                            if constexpr (kP16) {
                                umma::mma_f16_ts(tmem + kColO, tmem + kColP + 8 * j, b, idesc_o,
                                                 (i > 0 || j > 0) ? 1u : 0u);
                            } else {
                                umma::mma_f16_ts(tmem + kColO, pb + 16 * j, b, idesc_o,
                                                 (i > 0 || j > 0) ? 1u : 0u);
                                umma::mma_f16_ts(tmem + kColO, pb + 16 * j + 8, b, idesc_o, 1u);
                            }
                        }
                        umma::commit(pv_done + 8 * (gi & 1));
                        umma::commit(v_empty + 8 * slot);
                    }
                }
                ++tp;
            }
            if (!ok) {
                raise_device_error(p.err, PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            umma::commit(mma_done);  // arrives when every MMA this thread issued is done
        }
        return;
    }

    // ------------------------------------------------------------ softmax warps
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;  // row == TMEM lane
    const int tl = r / G, hh = r - tl * G;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    // S is computed with sign(scale) folded into Q (a sign-bit flip, exact),
    // so that the logit scale applied below is non-negative
    const uint32_t qflip = p.scale_log2 < 0.f ? 0x80008000u : 0u;
    const float sl2 = fabsf(p.scale_log2);
    // the tile's row: the row's last key position, the tile's key count
    int qp = 0, nkeys = 0;
    // The Q row of a tile, two elements per 32-bit word: for D 128 each half
    // of the row's threads takes 32 words, for D 64 the first takes all.
    // Loaded into registers first, so that the loads of the next tile's Q
    // can be in flight while the current tile's output is written.
    const bool q_writer = D == 128 || half == 0;
    const bool out32 = (reinterpret_cast<uintptr_t>(p.out) & 31u) == 0;
    auto load_q = [&](const Tile &t, uint32_t (&w)[32]) {
        const bool ok_row = r < TQ * G && tl < t.ntok;
        const int64_t row = ((int64_t)(t.q0 + t.tok0 + tl) * p.num_heads + t.g * G + hh) * D;
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const T *>(p.q) + row) +
                           half * (D == 128 ? 8 : 0);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint4 v = ok_row && q_writer ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
            w[4 * c] = v.x ^ qflip;
            w[4 * c + 1] = v.y ^ qflip;
            w[4 * c + 2] = v.z ^ qflip;
            w[4 * c + 3] = v.w ^ qflip;
        }
    };
    // into TMEM buffer b, then counted on that buffer's q_full barrier
    auto store_q = [&](uint32_t (&w)[32], int b) {
        if (q_writer) {
            umma::st32(lane_base + kColQ + b * (D / 2) + half * 32, w);
            umma::wait_st();
        }
        umma::fence_before_sync();
        mbar_arrive(q_full + 8 * b);
    };
    float *xch = reinterpret_cast<float *>(smem + C::kXchOffset);  // [parity][half][row]
    const uint32_t my_xchg = xchg + 8 * quarter;
    int xp = 0;  // exchanges so far (the same sequence for both threads of a row)
    // the partner thread's value of x (same row, other half of the keys)
    auto exchange = [&](float x, float &other) -> bool {
        xch[((xp & 1) * 2 + half) * kM + r] = x;
        mbar_arrive(my_xchg);
        const bool got = __all_sync(0xffffffffu, mbar_wait_bounded(my_xchg, xp & 1, abort_flag));
        other = xch[((xp & 1) * 2 + (half ^ 1)) * kM + r];
        ++xp;
        return got;
    };
    float m = -INFINITY, l = 0.f;
    // One stage.  Stages reaching beyond the first chunk token run the
    // masked body, every earlier stage the unmasked one.
    auto stage = [&](int i, int gi, auto masked_c) __attribute__((always_inline)) -> bool {
        constexpr bool kMasked = decltype(masked_c)::value;
        if (!warp_wait(s_full + 8 * (gi & 1), (gi >> 1) & 1, abort_flag)) return false;
        umma::fence_after_sync();
        const uint32_t hcol = lane_base + (gi & 1) * kKeys + half * 64;  // this thread's S / P
        const int last = qp - (i * kKeys + half * 64);  // the row's last key in the half
        uint32_t sr[2][32];
        umma::ld32(hcol, sr[0]);
        umma::ld32(hcol + 32, sr[1]);
        umma::wait_ld();
        float mx;
        {
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    if constexpr (kMasked) {
                        const float v = 32 * c + e > last ? -INFINITY : __uint_as_float(sr[c][e]) * sl2;
                        m4[e & 3] = fmaxf(m4[e & 3], v);
                    } else if (e % 2 == 0) {
                        m4[(e >> 1) & 3] = max3(m4[(e >> 1) & 3], __uint_as_float(sr[c][e]),
                                                __uint_as_float(sr[c][e + 1]));
                    }
                }
            mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            if constexpr (!kMasked) mx *= sl2;  // sl2 >= 0
        }
        float other;
        if (!exchange(mx, other)) return false;
        mx = fmaxf(mx, other);
        // the running max moves only when it grows by more than 8 (log2 units):
        // weights then stay below 2^8 and O is rescaled rarely
        float alpha = 1.f;
        bool rescale = false;
        if (mx > m + 8.f) {
            alpha = umma::ex2(m - mx);  // 0 on the first stage (m = -inf)
            rescale = m != -INFINITY;
            m = mx;
        }
        // weights 2^(x - m), summed and split in place: the pair of keys
        // (2e, 2e+1) of a 32-key chunk leaves its high-part word in word 2e
        // and its remainder word in word 2e+1; the chunk's TMEM column q then
        // takes key block q / 16 of the chunk, high parts in its first 8
        // columns, remainders in the next 8 (over the chunk's own S columns)
        uint64_t acc[2] = {pk(0.f, 0.f), pk(0.f, 0.f)};
        // (the one-fp16 form: the pair's word is word 16c + e of the thread's
        // 32 P columns, kColP + 32 half: key block j of the tile at kColP + 8 j)
        [[maybe_unused]] uint32_t p16[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint32_t(&w)[32] = sr[c];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                float y0 = fmaf(__uint_as_float(w[2 * e]), sl2, -m);
                float y1 = fmaf(__uint_as_float(w[2 * e + 1]), sl2, -m);
                if constexpr (kMasked) {
                    if (32 * c + 2 * e > last) y0 = -INFINITY;
                    if (32 * c + 2 * e + 1 > last) y1 = -INFINITY;
                }
                const float p0 = umma::ex2(y0), p1 = umma::ex2(y1);
                acc[e & 1] = add2(acc[e & 1], pk(p0, p1));
                if constexpr (kP16)
                    p16[16 * c + e] = Mma<__half>::pack(p0, p1);
                else
                    PSplit<T>::run(p0, p1, w[2 * e], w[2 * e + 1]);
            }
            if constexpr (!kP16) {
                uint32_t pw[32];
#pragma unroll
                for (int q = 0; q < 32; ++q)
                    pw[q] = w[2 * ((q >> 4) * 8 + (q & 7)) + ((q >> 3) & 1)];
                umma::st32(hcol + 32 * c, pw);
            }
        }
        if constexpr (kP16) {
            // P(gi) goes where P(gi-1) was: once PV(gi-1) has read it
            if (i > 0 && !warp_wait(pv_done + 8 * ((gi - 1) & 1), ((gi - 1) >> 1) & 1, abort_flag))
                return false;
            umma::fence_after_sync();
            umma::st32(lane_base + kColP + half * 32, p16);
        }
        {
            float a0, a1, b0, b1;
            upk(acc[0], a0, a1);
            upk(acc[1], b0, b1);
            l = l * alpha + ((a0 + a1) + (b0 + b1));
        }
        if (__any_sync(0xffffffffu, rescale)) {  // warp-collective TMEM access
            // O must hold PV up to stage i-1 before it is rescaled
            if (i > 0 && !warp_wait(pv_done + 8 * ((gi - 1) & 1), ((gi - 1) >> 1) & 1, abort_flag))
                return false;
            umma::fence_after_sync();
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
                uint32_t o[32];
                const uint32_t col = lane_base + kColO + half * (D / 2) + 32 * cb;
                umma::ld32(col, o);
                umma::wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                umma::st32(col, o);
            }
        }
        if constexpr (kMasked && !kConv) {  // (the converters zero them in that form)
            if (i * kKeys + kKeys > nkeys) {
                // last stage: V rows past the last key hold stale or unwritten
                // data; zero them so that their zero weights give exact zeros.
                // The wait only orders these stores after the stage's copies.
                if (!warp_wait(v_full + 8 * (gi % NV), (gi / NV) & 1, abort_flag)) return false;
                const int first = nkeys - i * kKeys;  // rows [first, 128)
                uint8_t *vst = smem + C::kVOffset + (gi % NV) * C::kStageBytes;
                for (int idx = threadIdx.x; idx < (kKeys - first) * C::kPieces * 8;
                     idx += kSoftmaxThreads) {
                    const int row = first + idx / (C::kPieces * 8);
                    const int rem = idx % (C::kPieces * 8);
                    *reinterpret_cast<uint4 *>(vst + (rem >> 3) * C::kKVPiece + row * kRowBytes +
                                               ((rem & 7) << 4)) = make_uint4(0u, 0u, 0u, 0u);
                }
                umma::fence_proxy_async_smem();
            }
        }
        umma::wait_st();
        umma::fence_before_sync();
        mbar_arrive(p_full + 8 * (gi & 1));
        return true;
    };
    // The CTA's tiles in turn.  Between two tiles: the next tile's Q loads go
    // out, the last PV of the tile is waited for, the next Q goes into the
    // other TMEM buffer (so the S thread can start the next tile while this
    // one's output is written), O is read out and o_free counted, and the
    // output is normalised and stored.
    bool ok = true;
    int gi = 0, tp = 0;  // stages and tiles done, the same counts as the MMA threads'
    Tile t;
    int u = u0;
    bool have = false;
    for (; !have && u < ntiles; u += have ? 0 : ustep)
        have = describe_tile<BS, kPersist>(p, u, threadIdx.x == 0, t);
    if (have) {
        uint32_t w[32];
        load_q(t, w);
        store_q(w, 0);
    }
    while (have && ok) {
        const bool valid = r < TQ * G && tl < t.ntok;
        qp = valid ? t.pos0 + tl : t.nkeys - 1;
        nkeys = t.nkeys;
        // stages i < n_fast end at or before the first chunk token: no mask there
        const int n_fast = min(t.nstages, (t.pos0 + 1) / kKeys);
        m = -INFINITY;
        l = 0.f;
        int i = 0;
        for (; ok && i < n_fast; ++i) ok = stage(i, gi + i, std::false_type{});
        for (; ok && i < t.nstages; ++i) ok = stage(i, gi + i, std::true_type{});
        if (!ok) break;
        const int glast = gi + t.nstages - 1;
        gi += t.nstages;
        // the next tile, if any
        Tile nt;
        bool have_next = false;
        int un = u + ustep;
        for (; !have_next && un < ntiles; un += have_next ? 0 : ustep)
            have_next = describe_tile<BS, kPersist>(p, un, threadIdx.x == 0, nt);
        uint32_t w[32];
        if (have_next) load_q(nt, w);
        float other = 0.f;
        ok = warp_wait(pv_done + 8 * (glast & 1), (glast >> 1) & 1, abort_flag) &&
             exchange(l, other);
        if (!ok) break;
        umma::fence_after_sync();
        if (have_next) store_q(w, (tp + 1) & 1);
        const float lt = l + other;
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const int64_t qrow = ((int64_t)(t.q0 + t.tok0 + tl) * p.num_heads + t.g * G + hh) * D;
        float *dst = p.out + qrow + half * (D / 2);
        // O out of TMEM a 32-column chunk at a time, normalised and stored;
        // each lane writes its own row: 32-byte stores when out allows them
        // (whole sectors), else 16-byte ones
        [[maybe_unused]] uint32_t nonfinite = 0u;
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb) {
            uint32_t o[32];
            umma::ld32(lane_base + kColO + half * (D / 2) + 32 * cb, o);
            umma::wait_ld();
            if constexpr (kConv) {
                // a V value beyond the fp16 range became infinite in the
                // conversion and reaches every row of the tile
#pragma unroll
                for (int e = 0; e < 32; ++e) nonfinite |= (~o[e] & 0x7f800000u) == 0u;
            }
            if (cb == D / 64 - 1) {
                // O is out of TMEM: the next tile's first PV may start it afresh
                umma::fence_before_sync();
                mbar_arrive(o_free);
            }
            if (valid && out32) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    float v8[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) v8[k] = __uint_as_float(o[e + k]) * inv;
                    st_global_v8(dst + cb * 32 + e, v8);
                }
            } else if (valid) {
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(dst + cb * 32 + e) = make_float4(
                        __uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv,
                        __uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
            }
        }
        if constexpr (kConv) {
            if (valid && nonfinite) raise_device_error(p.err, PA_DEVERR_RANGE);
        }
        ++tp;
        t = nt;
        u = un;
        have = have_next;
    }
    if (!ok && lane == 0) {
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

template <typename T, int D, int BS, bool kPersist, bool kP16>
static cudaError_t launch_inst(const PrefillParams &p, const CUtensorMap &mk,
                               const CUtensorMap &mv, cudaStream_t stream) {
    constexpr int NK = D == 128 ? 3 : 6, NV = D == 128 ? 3 : 6;
    using C = Cfg<D, BS, NK, NV>;
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(prefill_umma_kernel<T, D, BS, NK, NV, kPersist, kP16>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kDynSmem);
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];
    const int tiles_x = (p.max_q_len + p.tokens_per_cta - 1) / p.tokens_per_cta;
    cudaLaunchConfig_t cfg = {};
    if constexpr (kPersist) {
        // one CTA per SM (shared memory and TMEM allow no more), each walking
        // its share of the tile list
        const int64_t tiles = (int64_t)tiles_x * p.num_kv_heads * p.num_seqs;
        if (tiles > INT_MAX) return cudaErrorInvalidValue;
        const int sms = num_sms();
        if (sms <= 0) return cudaErrorInvalidDevice;
        cfg.gridDim = dim3((unsigned)std::min<int64_t>(tiles, sms));
    } else {
        cfg.gridDim = dim3(tiles_x, p.num_kv_heads, p.num_seqs);
    }
    cfg.blockDim = dim3(threads_for(kP16 && std::is_same<T, __nv_bfloat16>::value));
    cfg.dynamicSmemBytes = C::kDynSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_umma_kernel<T, D, BS, NK, NV, kPersist, kP16>, mk, mv,
                              p);
}

template <typename T, int D, bool kPersist, bool kP16>
static cudaError_t launch_d(const PrefillParams &p, const CUtensorMap &mk, const CUtensorMap &mv,
                            cudaStream_t stream) {
    switch (p.block_size) {
    case 8: return launch_inst<T, D, 8, kPersist, kP16>(p, mk, mv, stream);
    case 16: return launch_inst<T, D, 16, kPersist, kP16>(p, mk, mv, stream);
    case 32: return launch_inst<T, D, 32, kPersist, kP16>(p, mk, mv, stream);
    case 64: return launch_inst<T, D, 64, kPersist, kP16>(p, mk, mv, stream);
    default: return cudaErrorNotSupported;
    }
}

// form 0: one tile per CTA; 1: persistent; 2: one tile per CTA, P as one
// fp16 per weight (a bf16 cache's V stages converted to fp16)
template <typename T, int D>
static cudaError_t launch_p(const PrefillParams &p, int form, const CUtensorMap &mk,
                            const CUtensorMap &mv, cudaStream_t stream) {
    if (form == 1) return launch_d<T, D, true, false>(p, mk, mv, stream);
    if (form == 2) return launch_d<T, D, false, true>(p, mk, mv, stream);
    return launch_d<T, D, false, false>(p, mk, mv, stream);
}

}  // namespace pu

cudaError_t launch_prefill_umma(const PrefillParams &p, int dtype, int form,
                                cudaStream_t stream) {
    if (p.num_seqs == 0 || p.max_q_len == 0) return cudaSuccess;
    const int64_t rows = (int64_t)p.num_blocks * p.num_kv_heads * p.block_size;
    CUtensorMap mk, mv;
    if (!make_cache_tensor_map(&mk, p.k_cache, dtype, p.head_dim, rows, p.block_size) ||
        !make_cache_tensor_map(&mv, p.v_cache, dtype, p.head_dim, rows, p.block_size))
        return cudaErrorInvalidValue;
    if (dtype == PA_BF16)
        return p.head_dim == 128 ? pu::launch_p<__nv_bfloat16, 128>(p, form, mk, mv, stream)
                                 : pu::launch_p<__nv_bfloat16, 64>(p, form, mk, mv, stream);
    return p.head_dim == 128 ? pu::launch_p<__half, 128>(p, form, mk, mv, stream)
                             : pu::launch_p<__half, 64>(p, form, mk, mv, stream);
}

}  // namespace pa
