// Masked spatio-temporal attention forward on tcgen05 tensor cores (libvdit, sm_100a).
//
// Computes o = softmax(R(p_q) q . R(p_k) k * scale, restricted to the mask) v for every
// (query block, head) of a plan: the O(N^2) step of full spatio-temporal attention ("Accelerating
// Video Generation Inference with Sequential-Parallel 3D Positional Encoding Using a Global Time
// Index", section 1) over the block-causal / radial tile schedule ("DynamicRad", section 2;
// Wave Forcing / WaveRT block-causal chunks). Only the tiles the plan lists are visited; a tile
// flagged full needs no mask; a partial one applies the per-row keep bits the plan computed.
//
// One CTA = two 128-row query tiles (Q0, Q1) of one head, sharing every K/V tile it loads, over
// the union list of the two tiles' entries or, where the plan's CTA schedule cut the unit, one
// key piece of it (its normalised fp32 partial result then goes to a workspace slot and
// split_combine_kernel merges the pieces); 12 warps (3 warpgroups):
//   warps 0-3   softmax of Q0, warps 4-7 softmax of Q1: thread r owns query row r (TMEM lane r);
//               tcgen05.ld of its S row (after which the S columns are released), mask, online
//               softmax in fp32 (log2 domain; O is rescaled in TMEM only when the running max
//               grows by more than 2^8), P written as bf16 into the group's own P columns of
//               TMEM (tcgen05.st), epilogue (O / l -> bf16, staged through shared memory for
//               256-byte coalesced row stores; natural-log LSE);
//   warp 8      producer: TMA (cp.async.bulk.tensor, SWIZZLE_128B) of K and V tiles from the
//               head-major cache into 2-stage rings, plus (bulk copy) the plan's per-row keep
//               masks of the partial tiles;
//   warp 9      TMEM allocator (512 columns) and the thread issuing the score MMAs, kind::f16
//               bf16 x bf16 -> fp32, M = 128: S_h = Q_h K^T (SS, N = 128) into the shared S
//               columns [0, 128). A score tile waits only until the previous one has been read
//               out of TMEM, so the tensor core computes the next scores of a group while that
//               group's softmax still works on the current tile;
//   warp 10     the thread issuing O_h += P_h V (TS: P_h from TMEM columns [128 + 64h, ..), V
//               the MN-major smem operand) into [256 + 128h, ..), as soon as P_h is stored
//               (warp 11 idle).
// Q is read from global memory, rotated (3-D RoPE at the plan's query positions, fp32 math on
// fp64-built tables) and written straight into the swizzled K-major layout the MMA reads: the
// RoPE of Q is fused into the Q load.
//
// Ordering: a score tile is issued after an mbarrier on which the previous tile's softmax group
// arrives once its tcgen05.ld has completed (wait::ld, fence::before_thread_sync); softmax h
// overwrites P_h and rescales O_h only after the commit of PV_h of its previous tile has
// arrived (tcgen05.commit signals when every earlier tcgen05 operation of the issuing thread has
// completed).
//
// Every mbarrier wait is bounded (globaltimer): on expiry the thread raises the CTA abort flag
// and the device status word (VDIT_ERR_TIMEOUT), every role leaves its loop, in-flight TMA and
// MMA work is drained (again bounded) and TMEM is freed before the CTA exits.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <string>
#include <type_traits>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sm100.h"

namespace {

constexpr int kTile = 128;
constexpr int kStages = 2;
constexpr int kQTiles = 2;                       // query tiles per CTA (one softmax group each)
constexpr int kSoftmaxThreads = 128 * kQTiles;
constexpr int kWarpTMA = 8, kWarpMMA = 9, kWarpPV = 10;  // warp 11 completes the third warpgroup
constexpr int kThreads = 384;
// Register split (setmaxnreg, per warpgroup): launched at 168 per thread (3 warps per SM
// sub-partition, 16384 registers each); the two softmax groups grow to 208 and the producer /
// MMA group shrinks to 88: 2 * 128 * 208 + 128 * 88 = 64512 = 384 * 168. (No call may sit
// inside a setmaxnreg region: the bounded wait is inlined.)
constexpr int kRegsSoftmax = 208, kRegsOther = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther == kThreads * 168, "register split");
constexpr uint32_t kSlabBytes = kTile * 64 * 2;  // 16 KiB: 128 rows x 128 B (one swizzle width)
// TMEM columns: S [0, 128) shared by the two query tiles, P0 [128, 192), P1 [192, 256) (bf16
// pairs), O0 [256, 384), O1 [384, 512).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemP = 128, kTmemO = 256;
constexpr float kRescaleTau = 8.0f;              // rescale O only when the max grows by > 2^8


// barrier indices (8 bytes each)
enum {
    B_KFULL = 0, B_KEMPTY = B_KFULL + kStages, B_VFULL = B_KEMPTY + kStages,
    B_VEMPTY = B_VFULL + kStages, B_IFULL = B_VEMPTY + kStages, B_IEMPTY = B_IFULL + kStages,
    B_SFULL = B_IEMPTY + kStages, B_SFREE = B_SFULL + kQTiles, B_PFULL = B_SFREE + 1,
    B_PVDONE = B_PFULL + kQTiles, B_DRAIN = B_PVDONE + kQTiles,
    B_SFREE1 = B_DRAIN + 1,  // dynamic-threshold logit pass: the second score buffer
    B_COUNT
};
static_assert(B_COUNT <= 32, "barrier area too small");
// Stage of the keep masks, one per K stage: a 16-byte header {tile, flags} and, for each query
// tile whose entry is partial, its 2 KiB block of per-row keep masks (128 rows x 4 words, bit k of
// row r: key k kept for query r), copied from the plan by the producer.
constexpr uint32_t kMaskBlockBytes = kTile * 16;
constexpr uint32_t kKinfoBytes = 16 + kQTiles * kMaskBlockBytes;

// Shared-memory map for head_dim D (offsets from a 1024-byte aligned base).
template <int D>
struct Layout {
    static constexpr int kSlabs = D / 64;
    static constexpr uint32_t kTileBytes = kTile * D * 2;  // one Q, K or V tile
    static constexpr uint32_t OFF_Q = 0;                   // kQTiles tiles
    static constexpr uint32_t OFF_K = OFF_Q + kQTiles * kTileBytes;
    static constexpr uint32_t OFF_V = OFF_K + kStages * kTileBytes;
    static constexpr uint32_t OFF_BAR = OFF_V + kStages * kTileBytes;
    static constexpr uint32_t OFF_MISC = OFF_BAR + 8 * 32;  // [0] tmem base, [1] abort flag
    static constexpr uint32_t OFF_KINFO = OFF_MISC + 64;
    static constexpr uint32_t kSmemBytes = OFF_KINFO + kStages * kKinfoBytes + 1024;  // + align slack
    static_assert(OFF_KINFO % 16 == 0 && kKinfoBytes % 16 == 0, "bulk-copy destinations 16-byte aligned");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

struct AttnArgs {
    const int* u_row_ptr;  // per block of two q-tiles: union list of key tiles
    const int* u_col;      // first key row of each entry (a multiple of 128, or the unaligned
                           // row of a single-patch entry)
    const unsigned char* u_flags;
    const int* cta;        // per CTA, 4 ints: q-block, head, first union entry of its piece, entries
    const int* cta_slot;   // per CTA: partial slot of a piece of a cut unit, or -1
    float* ws_o;           // normalised partial O of the pieces [slot][256 query rows][D]
    float* ws_lse;         // their log2-sum-exp [slot][256 query rows]
    const uint32_t* masks; // keep-mask blocks of the partial tiles (2 KiB each)
    const int* u_mask;     // per union entry and query tile: mask block, or -1
    const uint4* q;
    uint4* o;
    float* lse;
    const float2* tt;
    const float2* th;
    const float2* tw;
    int* status;
    int q_rotated;         // q already rotated at the plan's query positions: plain load
    int skip_loads;        // test hook: the producer issues nothing, so every wait runs out
    int bt2, bh2, bw2;
    int q_tokens, kv_tokens, heads;
    int grid_h, grid_w;
    int q_start;
    float scale_log2;
    float tau_log2;        // dynamic-threshold mode: tau * log2(e)
};

// ------------------------------------------------------------------------------ PTX wrappers


__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}


__device__ __forceinline__ uint4 rope_chunk(uint4 in, int pp0, int t, int h, int w,
                                            const AttnArgs& a) {
    uint32_t word[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int pp = pp0 + i;
        // band of this pair, chosen without branches: the lanes of a warp hold different
        // chunks of a head row and would otherwise split over the three table lookups
        const bool in_h = pp >= a.bt2, in_w = pp >= a.bt2 + a.bh2;
        const float2* tab = in_w ? a.tw : (in_h ? a.th : a.tt);
        const int row = in_w ? w : (in_h ? h : t);
        const int width = in_w ? a.bw2 : (in_h ? a.bh2 : a.bt2);
        const int jj = pp - (in_w ? a.bt2 + a.bh2 : (in_h ? a.bt2 : 0));
        const float2 cs = __ldg(tab + (size_t)row * width + jj);
        __nv_bfloat162 b;
        memcpy(&b, &word[i], 4);
        const float2 x = __bfloat1622float2(b);
        b = __floats2bfloat162_rn(fmaf(x.x, cs.x, -x.y * cs.y), fmaf(x.x, cs.y, x.y * cs.x));
        memcpy(&word[i], &b, 4);
    }
    return make_uint4(word[0], word[1], word[2], word[3]);
}


// ------------------------------------------------------------------------------ the kernel

template <int D, bool DYN>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const AttnArgs a) {
    using L = Layout<D>;
    constexpr uint32_t kTileBytes = L::kTileBytes;
    constexpr int kC16 = D / 8;  // 16-byte chunks per head row
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    auto BAR = [&](int i) { return sbase + L::OFF_BAR + 8u * (uint32_t)i; };
    volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // work of this CTA (the plan's schedule): q-block, head and a piece of the union list, whole
    // or cut; a piece of a cut unit writes partial results into its slot
    // (scalar loads: a 16-byte vector load here costs the kernel register spills)
    const int* work = a.cta + 4 * blockIdx.x;
    const int qb = __ldg(work), head = __ldg(work + 1);
    const int u_begin = __ldg(a.u_row_ptr + qb) + __ldg(work + 2);
    const int n_ent = __ldg(work + 3);
    const int unit = blockIdx.x;
    // Every CTA walks its key tiles starting at a different position (the online softmax does
    // not depend on the order): CTAs of one head run concurrently, and starting them all at the
    // same tile makes them request the same 32 KiB of K / V from the same L2 slices at once.
    const int rot = n_ent > 0 ? (int)(((unsigned)unit * 97u + (unsigned)head * 31u) % (unsigned)n_ent) : 0;
    auto entry = [&](int i) { const int e = i + rot; return e >= n_ent ? e - n_ent : e; };
    // visits of the entries: the dynamic-threshold mode walks the list twice
    const int n_v = DYN ? 2 * n_ent : n_ent;
    const int ft = a.grid_h * a.grid_w;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(BAR(B_KFULL + s), 1);
            mbar_init(BAR(B_KEMPTY + s), 1);
            mbar_init(BAR(B_VFULL + s), 1);
            mbar_init(BAR(B_VEMPTY + s), 1);
            mbar_init(BAR(B_IFULL + s), 1);
            mbar_init(BAR(B_IEMPTY + s), kSoftmaxThreads);
        }
        for (int h = 0; h < kQTiles; ++h) {
            mbar_init(BAR(B_SFULL + h), 1);
            mbar_init(BAR(B_PFULL + h), 128);
            mbar_init(BAR(B_PVDONE + h), 1);
        }
        mbar_init(BAR(B_SFREE), 128);
        mbar_init(BAR(B_SFREE1), 128);
        mbar_init(BAR(B_DRAIN), 2);  // one commit from each MMA-issuing thread
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         sbase + L::OFF_MISC),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // radius table and the two rotated Q tiles (all threads)
    for (int idx = threadIdx.x; idx < kQTiles * kTile * kC16; idx += kThreads) {
        const int h = idx / (kTile * kC16), rem = idx - h * (kTile * kC16);
        const int r = rem / kC16, c16 = rem - r * kC16;
        const int qi = (qb * kQTiles + h) * kTile + r;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (qi < a.q_tokens) {
            const int f = qi / ft, rm = qi - f * ft;
            const int hh = rm / a.grid_w, ww = rm - hh * a.grid_w;
            const uint4 x = __ldg(a.q + ((size_t)qi * a.heads + head) * kC16 + c16);
            v = a.q_rotated ? x : rope_chunk(x, c16 * 4, a.q_start + f, hh, ww, a);
        }
        *reinterpret_cast<uint4*>(smem + L::OFF_Q + h * kTileBytes + sw128_offset(r, c16)) = v;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp < 4 * kQTiles) {
        // ------------------------------------------------------------------ softmax (group h)
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        const int h = warp >> 2;
        const int row = threadIdx.x & 127;  // TMEM lane == query row within the tile
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + lane_base;
        const uint32_t t_p = tmem + kTmemP + 64u * h + lane_base;
        const uint32_t t_o = tmem + kTmemO + 128u * h + lane_base;
        const uint32_t f_in = h ? 4u : 1u, f_full = h ? 8u : 2u;
        const float c = a.scale_log2;
        float m = -INFINITY, l = 0.f;  // running max (raw score units) and sum
        int cnt = 0;                   // score tiles read
        int npv_dyn = 0;               // dynamic-threshold mode: P tiles stored (else == cnt)
        bool ok = true;
        // One score tile of the union list (entry j): P = 0 the attention tile of the static mask,
        // P = 1 the logit pass and P = 2 the attention pass of the dynamic-threshold mode. The
        // dynamic mode runs the two passes as two loops, so each loop body is compiled for its
        // pass alone (one body for both spilled registers in the loop). false: a wait ran out.
        auto score_tile = [&](const int j, auto pass) -> bool {
            // dynamic-threshold mode: pass 0 (j < n_ent) only takes the row maxima of the
            // candidates' logits; pass 1 keeps a candidate iff its logit is within tau of it
            constexpr bool pass0 = decltype(pass)::value == 1, pass1 = decltype(pass)::value == 2;
            const int npv = DYN ? npv_dyn : cnt;
            const int s = j % kStages;
            if (!warp_wait(BAR(B_IFULL + s), (j / kStages) & 1, abort_flag, a.status)) { ok = false; return false; }
            const uint8_t* info = smem + L::OFF_KINFO + s * kKinfoBytes;
            const uint32_t flags = (uint32_t)reinterpret_cast<const int*>(info)[1];
            // dynamic-threshold logit pass: each query tile's score tiles have a buffer of their own
            const uint32_t sbuf = pass0 ? (uint32_t)h : 0u;
            if (!(flags & f_in)) {
                mbar_arrive(BAR(B_IEMPTY + s));
                return true;
            }
            if (!warp_wait(BAR(B_SFULL + h), cnt & 1, abort_flag, a.status)) { ok = false; return false; }
            tc_fence_after();
            uint32_t sr[128];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(t_s + 128u * sbuf + q4 * 32, sr + q4 * 32);
            tmem_ld_wait(sr);
            reg_touch32(sr + 32);
            reg_touch32(sr + 64);
            reg_touch32(sr + 96);
            // S is in registers: the shared S columns may take the next score tile
            tc_fence_before();
            mbar_arrive(BAR(sbuf ? B_SFREE1 : B_SFREE));
            float* sv = reinterpret_cast<float*>(sr);
            if (!(flags & f_full)) {
                // this row's keep bits for the 128 keys of the tile, from the plan's mask block
                const uint4 km = *reinterpret_cast<const uint4*>(info + 16 + h * kMaskBlockBytes + row * 16);
                const uint32_t mw[4] = {km.x, km.y, km.z, km.w};
#pragma unroll
                for (int jj = 0; jj < 128; ++jj)
                    sv[jj] = ((mw[jj >> 5] >> (jj & 31)) & 1u) ? sv[jj] : -INFINITY;
            }
            mbar_arrive(BAR(B_IEMPTY + s));
            float m_tile = -INFINITY;
            if constexpr (pass1) {
                // the row maximum m is final; the threshold is applied in the exponent below
            } else {
                // row max: 8 independent chains of 3-input max
                float mx[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mx[i] = sv[i];
#pragma unroll
                for (int jj = 8; jj < 128; jj += 16) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) mx[i] = max3(mx[i], sv[jj + 2 * i], sv[jj + 2 * i + 1]);
                }
                m_tile = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
            }
            if constexpr (pass0) {
                m = fmaxf(m, m_tile);
                ++cnt;
                return true;
            }
            const float m_new = fmaxf(m, m_tile);
            const bool resc = (m_new - m) * c > kRescaleTau;
            float alpha = 1.f;
            if (resc) {
                alpha = fast_exp2((m - m_new) * c);
                m = m_new;
            }
            const float mc = (m == -INFINITY) ? 0.f : m * c;
            // PV_h of the previous tile must have completed: it reads P_h (overwritten below)
            // and accumulates into O_h (rescaled below)
            if (npv > 0) {
                if (!warp_wait(BAR(B_PVDONE + h), (npv - 1) & 1, abort_flag, a.status)) { ok = false; return false; }
                tc_fence_after();
            }
            if (npv > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
                for (int q4 = 0; q4 < D / 32; ++q4) {
                    uint32_t orow[32];
                    tmem_ld32(t_o + q4 * 32, orow);
                    tmem_ld_wait(orow);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        orow[i] = __float_as_uint(__uint_as_float(orow[i]) * alpha);
                    tmem_st32(t_o + q4 * 32, orow);
                }
            }
            // P = 2^(s*c - m*c) as bf16 pairs into the P_h columns of this lane (MUFU ex2)
            uint64_t rs2[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) rs2[i] = pack2(0.f, 0.f);
            const uint64_t c2 = pack2(c, c), nmc2 = pack2(-mc, -mc);
            // dynamic-threshold attention pass: a candidate is kept iff s c + (tau_log2 - m c) >= 0
            // (its logit within tau of the row maximum). z = (s c + (tau_log2 - m c)) 2^64 is one
            // packed FMA from s; the power-of-two factor changes no rounding, so z >= 0 exactly
            // when that fp32 sum is. A kept candidate has z >= 0 >= x = s c - m c, so min(x, z) = x.
            // A dropped one has z < 0: unless its sum lies within 150 * 2^-64 (~1e-17) of 0, z is
            // below -150 and ex2.approx.ftz of min(x, z) is exactly 0; inside that band, far inside
            // the fp32 rounding of the logits themselves, its weight lies between 0 and the kept
            // one. Two instructions per pair fewer than a compare and a select per element.
            constexpr float kZ = 18446744073709551616.f;  // 2^64
            uint64_t cz2 = 0, bz2 = 0;
            if constexpr (pass1) {
                cz2 = pack2(c * kZ, c * kZ);
                bz2 = pack2((a.tau_log2 - mc) * kZ, (a.tau_log2 - mc) * kZ);
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const uint64_t s2 = pack2(sv[64 * half + 2 * i], sv[64 * half + 2 * i + 1]);
                    const uint64_t x2 = fma2(s2, c2, nmc2);
                    float x0, x1;
                    unpack2(x2, x0, x1);
                    if constexpr (pass1) {
                        float z0, z1;
                        unpack2(fma2(s2, cz2, bz2), z0, z1);
                        x0 = fminf(x0, z0);
                        x1 = fminf(x1, z1);
                    }
                    const uint64_t p2 = pack2(fast_exp2(x0), fast_exp2(x1));
                    rs2[i & 3] = add2(rs2[i & 3], p2);
                    float p0, p1;
                    unpack2(p2, p0, p1);
                    __nv_bfloat162 b = __floats2bfloat162_rn(p0, p1);
                    memcpy(&pk[i], &b, 4);
                }
                tmem_st32(t_p + 32 * half, pk);
            }
            float rsum;
            {
                const uint64_t a01 = add2(rs2[0], rs2[1]), a23 = add2(rs2[2], rs2[3]);
                float u0, u1;
                unpack2(add2(a01, a23), u0, u1);
                rsum = u0 + u1;
            }
            tmem_st_wait();
            l = l * alpha + rsum;
            tc_fence_before();
            mbar_arrive(BAR(B_PFULL + h));
            ++cnt;
            if (DYN) ++npv_dyn;
            return true;
        };
        if constexpr (DYN) {
            for (int j = 0; j < n_ent; ++j)
                if (!score_tile(j, std::integral_constant<int, 1>{})) break;
            if (ok)
                for (int j = n_ent; j < n_v; ++j)
                    if (!score_tile(j, std::integral_constant<int, 2>{})) break;
        } else {
            for (int j = 0; j < n_ent; ++j)
                if (!score_tile(j, std::integral_constant<int, 0>{})) break;
        }
        const int n_pv = DYN ? npv_dyn : cnt;
        if (ok && n_pv > 0) {
            if (!warp_wait(BAR(B_PVDONE + h), (n_pv - 1) & 1, abort_flag, a.status)) ok = false;
        }
        // every thread of the group reaches this barrier (aborted or not); any failure skips
        // the epilogue of the whole group
        int any_fail;
        asm volatile(
            "{\n\t.reg .pred p, q;\n\t"
            "setp.eq.u32 p, %1, 0;\n\t"
            "bar.red.or.pred q, %2, 128, p;\n\t"
            "selp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(any_fail)
            : "r"((uint32_t)ok), "r"(1 + h)
            : "memory");
        // the CTA's slot, q-block and head, read again here rather than kept live through the
        // loop (the softmax warps are short of registers)
        const int slot = __ldg(a.cta_slot + blockIdx.x);
        const int qb_e = __ldg(a.cta + 4 * blockIdx.x), head_e = __ldg(a.cta + 4 * blockIdx.x + 1);
        const int qi = (qb_e * kQTiles + h) * kTile + row;
        if (!any_fail && slot >= 0) {
            // partial result of this key piece: O / l in fp32 and log2(sum) for the merge
            tc_fence_after();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            const size_t prow = (size_t)slot * (kQTiles * kTile) + h * kTile + row;
            float4* dst = reinterpret_cast<float4*>(a.ws_o + prow * D);
#pragma unroll 1
            for (int q4 = 0; q4 < D / 32; ++q4) {
                uint32_t orow[32];
                if (n_pv > 0) {
                    tmem_ld32(t_o + q4 * 32, orow);
                    tmem_ld_wait(orow);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) orow[i] = 0u;
                }
                if (qi < a.q_tokens) {
#pragma unroll
                    for (int g = 0; g < 8; ++g)
                        dst[q4 * 8 + g] = make_float4(__uint_as_float(orow[4 * g]) * inv_l,
                                                      __uint_as_float(orow[4 * g + 1]) * inv_l,
                                                      __uint_as_float(orow[4 * g + 2]) * inv_l,
                                                      __uint_as_float(orow[4 * g + 3]) * inv_l);
                }
            }
            if (qi < a.q_tokens) a.ws_lse[prow] = l > 0.f ? m * c + log2f(l) : -INFINITY;
        } else if (!any_fail) {
            tc_fence_after();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            uint8_t* stage = smem + L::OFF_Q + h * kTileBytes;  // Q_h is no longer read
#pragma unroll 1
            for (int q4 = 0; q4 < D / 32; ++q4) {
                uint32_t orow[32];
                if (n_pv > 0) {
                    tmem_ld32(t_o + q4 * 32, orow);
                    tmem_ld_wait(orow);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) orow[i] = 0u;
                }
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t wds[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat162 b = __floats2bfloat162_rn(
                            __uint_as_float(orow[g * 8 + 2 * e]) * inv_l,
                            __uint_as_float(orow[g * 8 + 2 * e + 1]) * inv_l);
                        memcpy(&wds[e], &b, 4);
                    }
                    const int chunk = q4 * 4 + g;
                    *reinterpret_cast<uint4*>(stage + row * (D * 2) + ((chunk ^ (row & 7)) << 4)) =
                        make_uint4(wds[0], wds[1], wds[2], wds[3]);
                }
            }
            if (a.lse && qi < a.q_tokens)
                a.lse[(size_t)head_e * a.q_tokens + qi] =
                    l > 0.f ? (m * c + log2f(l)) * 0.6931471805599453f : -INFINITY;
            asm volatile("bar.sync %0, 128;" ::"r"(3 + h) : "memory");
            const int q0 = (qb_e * kQTiles + h) * kTile;
#pragma unroll 4
            for (int i = 0; i < kC16; ++i) {
                const int r = i * (128 / kC16) + row / kC16, chunk = row % kC16;
                if (q0 + r < a.q_tokens) {
                    const uint4 v = *reinterpret_cast<const uint4*>(stage + r * (D * 2) +
                                                                    ((chunk ^ (r & 7)) << 4));
                    __stcs(a.o + ((size_t)(q0 + r) * a.heads + head_e) * kC16 + chunk, v);
                }
            }
        }
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
    }
    if (warp == kWarpTMA) {
        // ------------------------------------------------------------------ producer
        // Pass 0 of the dynamic-threshold mode visits the entries for the logit maxima only (K
        // and masks); the attention pass loads K, masks and V. it: K / mask sequence number,
        // jv: V sequence number.
        // for the drain: last K and V sequence numbers issued, and per stage the last sequence
        // number whose masks were copied (scalars: the stage index is not a compile-time value)
        static_assert(kStages == 2, "drain bookkeeping assumes two stages");
        int k_last = -1, v_last = -1, mask_it0 = -1, mask_it1 = -1;
        auto load_entry = [&](int v, int& kt, int& fl, int& m0, int& m1) {
            const int e = u_begin + entry(DYN && v >= n_ent ? v - n_ent : v);
            kt = __ldg(a.u_col + e);
            fl = __ldg(a.u_flags + e);
            m0 = __ldg(a.u_mask + 2 * e);
            m1 = __ldg(a.u_mask + 2 * e + 1);
        };
        int kt_next = 0, fl_next = 0, mk0_next = -1, mk1_next = -1;
        if (n_ent > 0) load_entry(0, kt_next, fl_next, mk0_next, mk1_next);
        for (int it = 0; it < (a.skip_loads ? 0 : n_v); ++it) {
            const int s = it % kStages;
            const uint32_t ph = (uint32_t)((it / kStages) - 1) & 1u;
            const int kt = kt_next, flags = fl_next, mk0 = mk0_next, mk1 = mk1_next;
            // next entry's tile, flags and masks, loaded while this one waits
            if (it + 1 < n_v) load_entry(it + 1, kt_next, fl_next, mk0_next, mk1_next);
            if (it >= kStages && !warp_wait(BAR(B_KEMPTY + s), ph, abort_flag, a.status)) break;
            if (lane == 0) {
                mbar_expect_tx(BAR(B_KFULL + s), kTileBytes);
                const uint32_t dst = sbase + L::OFF_K + s * kTileBytes;
#pragma unroll
                for (int sl = 0; sl < L::kSlabs; ++sl)
                    tma_load_3d(dst + sl * kSlabBytes, &tmap_k, BAR(B_KFULL + s), 64 * sl, kt, head);
                k_last = it;
            }
            if (it >= kStages && !warp_wait(BAR(B_IEMPTY + s), ph, abort_flag, a.status)) break;
            uint8_t* info = smem + L::OFF_KINFO + s * kKinfoBytes;
            if (lane == 0) {
                reinterpret_cast<int*>(info)[0] = kt;
                reinterpret_cast<int*>(info)[1] = flags;
                // keep masks of the partial query tiles of this entry (2 KiB each), else a plain
                // arrival: the header above is published by the arrive's release either way
                const uint32_t nbytes = (mk0 >= 0 ? kMaskBlockBytes : 0u) + (mk1 >= 0 ? kMaskBlockBytes : 0u);
                if (nbytes) {
                    mbar_expect_tx(BAR(B_IFULL + s), nbytes);
                    const uint32_t dst = sbase + L::OFF_KINFO + s * kKinfoBytes + 16;
                    if (mk0 >= 0)
                        bulk_load(dst, a.masks + (size_t)mk0 * (kMaskBlockBytes / 4), kMaskBlockBytes, BAR(B_IFULL + s));
                    if (mk1 >= 0)
                        bulk_load(dst + kMaskBlockBytes, a.masks + (size_t)mk1 * (kMaskBlockBytes / 4),
                                  kMaskBlockBytes, BAR(B_IFULL + s));
                    if (s == 0) mask_it0 = it; else mask_it1 = it;
                } else {
                    mbar_arrive(BAR(B_IFULL + s));
                }
            }
            __syncwarp();
            if (DYN && it < n_ent) continue;  // logit pass: no V
            const int jv = DYN ? it - n_ent : it;
            const int sv = jv % kStages;
            if (jv >= kStages &&
                !warp_wait(BAR(B_VEMPTY + sv), (uint32_t)((jv / kStages) - 1) & 1u, abort_flag, a.status))
                break;
            if (lane == 0) {
                mbar_expect_tx(BAR(B_VFULL + sv), kTileBytes);
                const uint32_t dst = sbase + L::OFF_V + sv * kTileBytes;
#pragma unroll
                for (int sl = 0; sl < L::kSlabs; ++sl)
                    tma_load_3d(dst + sl * kSlabBytes, &tmap_v, BAR(B_VFULL + sv), 64 * sl, kt, head);
                v_last = jv;
            }
            __syncwarp();
        }
        // drain: every copy this warp issued must have landed before the CTA may exit
        if (*abort_flag && lane == 0) {
            auto drain = [&](int bar, int seq) {
                if (seq < 0) return;
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(BAR(bar + seq % kStages), (uint32_t)(seq / kStages) & 1u) &&
                       globaltimer() - t0 < kWaitLimitNs) {
                }
            };
            drain(B_IFULL, mask_it0);
            drain(B_IFULL, mask_it1);
            for (int x = k_last - kStages + 1; x <= k_last; ++x) drain(B_KFULL, x);
            for (int x = v_last - kStages + 1; x <= v_last; ++x) drain(B_VFULL, x);
        }
    } else if (warp == kWarpMMA || warp == kWarpPV) {
        // ------------------------------------------------------------------ MMA issuers
        // Two issuing threads: warp 9 issues the score MMAs, warp 10 the PV MMAs. Each waits
        // only for its own operands, so a wait of one never leaves the tensor core without
        // queued work from the other (an issuing thread that stops to poll an mbarrier, even
        // a completed one, leaves a gap in the tensor pipe).
        const bool s_role = warp == kWarpMMA;
        if (lane == 0 && n_ent > 0) {
            constexpr uint32_t idesc_qk = instr_desc(kTile, 0), idesc_pv = instr_desc(D, 1);
            // Descriptors are built once; each MMA only adds a compile-time offset (in 16-byte
            // units) to a loop-invariant base, which keeps the issuing thread at the tensor
            // core's rate (a descriptor rebuilt from runtime indices per MMA was measured to
            // cost more issue time than the 64-cycle M=128 N=128 K=16 MMA itself).
            const uint64_t dq0 = smem_desc_sw128(sbase + L::OFF_Q, 16, 1024);
            const uint64_t dk0 = smem_desc_sw128(sbase + L::OFF_K, 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(sbase + L::OFF_V, kSlabBytes, 1024);
            constexpr uint64_t kTileDesc = kTileBytes >> 4;  // one tile further, in descriptor units
            const unsigned char* fl = a.u_flags + u_begin;
            // tile flags are read two entries ahead so the global-load latency never sits
            // between a completed barrier and the next MMA issue
            auto flag_of = [&](int v) { return (int)__ldg(fl + entry(DYN && v >= n_ent ? v - n_ent : v)); };
            int f_cur = flag_of(0);
            int f_nxt = n_ent > 1 || DYN ? flag_of(1 % n_v) : 0;
            if (s_role) {
                // S_h(j) = Q_h K(j)^T into the shared S columns, in list order, each after the
                // previous score tile has been read out of TMEM by its softmax group
                int ns = 0;
                // dynamic-threshold logit pass: the P columns are idle, so each query tile's score
                // tiles get a buffer of their own (group h: [128 h, 128 h + 128)); a group's next
                // score tile waits only for its previous one to be read (never two unread, so a
                // group's SFULL phases cannot run two ahead of its waits). Uses of each buffer so
                // far, and whether buffer 1 has been drained before the first attention-pass tile
                int uses0 = 0, uses1 = 0;
                bool drained1 = false;
                for (int j = 0; j < n_v; ++j) {  // both passes in the dynamic-threshold mode
                    const int s = j % kStages;
                    const int f = f_cur;
                    f_cur = f_nxt;
                    f_nxt = j + 2 < n_v ? flag_of(j + 2) : 0;
                    if (!wait_bounded(BAR(B_KFULL + s), (j / kStages) & 1, abort_flag, a.status)) break;
                    tc_fence_after();
                    const uint64_t k0 = dk0 + (s ? kTileDesc : 0);
                    bool ok = true;
#pragma unroll
                    for (int h = 0; h < kQTiles; ++h) {
                        if (!(f & (h ? 4 : 1))) continue;
                        uint32_t sbuf = 0;
                        if (DYN) {
                            // the buffer's previous score tile has been read out
                            sbuf = j < n_ent ? (uint32_t)h : 0u;
                            const int uses = sbuf ? uses1 : uses0;
                            if (uses > 0) {
                                if (!wait_bounded(BAR(sbuf ? B_SFREE1 : B_SFREE), (uses - 1) & 1, abort_flag, a.status)) { ok = false; break; }
                            }
                            if (j >= n_ent && !drained1) {
                                // attention pass: the P columns must hold no unread score tile
                                if (uses1 > 0 &&
                                    !wait_bounded(BAR(B_SFREE1), (uses1 - 1) & 1, abort_flag, a.status)) { ok = false; break; }
                                drained1 = true;
                            }
                            if (sbuf) ++uses1; else ++uses0;
                            tc_fence_after();
                        } else if (ns > 0) {
                            if (!wait_bounded(BAR(B_SFREE), (ns - 1) & 1, abort_flag, a.status)) { ok = false; break; }
                            tc_fence_after();
                        }
                        const uint64_t q0 = dq0 + (h ? kTileDesc : 0);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t off = (uint64_t)((((kk >> 2) * kSlabBytes) + (kk & 3) * 32) >> 4);
                            tc_mma(tmem + 128u * sbuf, q0 + off, k0 + off, idesc_qk, kk > 0);
                        }
                        tc_commit(BAR(B_SFULL + h));
                        ++ns;
                    }
                    if (!ok) break;
                    tc_commit(BAR(B_KEMPTY + s));
                }
            } else {
                // O_h += P_h(j) V(j), each as soon as softmax h has stored P_h(j)
                int npv[2] = {0, 0};
                for (int j = 0; j < n_ent; ++j) {
                    const int s = j % kStages;
                    const int f = f_cur;
                    f_cur = f_nxt;
                    f_nxt = j + 2 < n_ent ? __ldg(fl + entry(j + 2)) : 0;
                    if (!wait_bounded(BAR(B_VFULL + s), (j / kStages) & 1, abort_flag, a.status)) break;
                    const uint64_t v0 = dv0 + (s ? kTileDesc : 0);
                    bool ok = true;
#pragma unroll
                    for (int h = 0; h < kQTiles; ++h) {
                        if (!(f & (h ? 4 : 1))) continue;
                        if (!wait_bounded(BAR(B_PFULL + h), npv[h] & 1, abort_flag, a.status)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t d_t = tmem + kTmemO + 128u * h;
                        const uint32_t a_t = tmem + kTmemP + 64u * h;
                        const uint32_t acc0 = npv[h] > 0 ? 1u : 0u;
#pragma unroll
                        for (int kk = 0; kk < kTile / 16; ++kk)
                            tc_mma_ts(d_t, a_t + 8u * kk, v0 + (uint64_t)((kk * 16 * 128) >> 4), idesc_pv,
                                      kk > 0 ? 1u : acc0);
                        tc_commit(BAR(B_PVDONE + h));
                        ++npv[h];
                    }
                    if (!ok) break;
                    tc_commit(BAR(B_VEMPTY + s));
                }
            }
        }
        if (lane == 0) {
            // drain: all MMAs issued by both threads complete before TMEM is released
            tc_commit(BAR(B_DRAIN));
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(BAR(B_DRAIN), 0) && globaltimer() - t0 < kWaitLimitNs) {
            }
        }
        __syncwarp();
    }
    // ---------------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
    }
}

// Merge of the key pieces of every cut unit's (query, head) rows: with piece i holding
// O_i = (sum over its keys of p v) / l_i and L_i = log2 l_i (in the shared log2 units of the
// scaled scores),
//   L = log2 sum_i 2^L_i,   o = sum_i 2^(L_i - L) O_i,   lse = L ln 2.
// merge[4 j ..] = q-block, head, first slot, pieces of cut unit j; its 256 query rows are rows
// 256 j .. 256 j + 255 of the grid-stride loop. One warp per row; each lane owns D / 32
// consecutive channels.
template <int D>
__global__ void __launch_bounds__(256) split_combine_kernel(const float* __restrict__ ws_o,
                                                            const float* __restrict__ ws_lse,
                                                            const int4* __restrict__ merge, int n_cut,
                                                            int q_tokens, int heads,
                                                            __nv_bfloat16* __restrict__ o,
                                                            float* __restrict__ lse) {
    constexpr int kPer = D / 32, kRows = kQTiles * kTile;
    const long long rows = (long long)n_cut * kRows;
    const long long n_warps = (long long)gridDim.x * (blockDim.x / 32);
    const int lane = threadIdx.x & 31;
    for (long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; row < rows;
         row += n_warps) {
        const int j = (int)(row / kRows), r = (int)(row - (long long)j * kRows);
        const int4 mu = __ldg(merge + j);
        const int qi = mu.x * kRows + r, hd = mu.y;
        if (qi >= q_tokens) continue;
        const size_t first = (size_t)mu.z * kRows + r;  // partial row of piece 0
        float lmax = -INFINITY;
        for (int i = 0; i < mu.w; ++i) lmax = fmaxf(lmax, __ldg(ws_lse + first + (size_t)i * kRows));
        float acc[kPer];
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
        float wsum = 0.f;
        if (lmax != -INFINITY) {
            for (int i = 0; i < mu.w; ++i) {
                const size_t prow = first + (size_t)i * kRows;
                const float w = exp2f(__ldg(ws_lse + prow) - lmax);
                wsum += w;
                const float* src = ws_o + prow * D + lane * kPer;
#pragma unroll
                for (int e = 0; e < kPer; ++e) acc[e] = fmaf(w, __ldg(src + e), acc[e]);
            }
        }
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
        __nv_bfloat16* dst = o + ((size_t)qi * heads + hd) * D + lane * kPer;
#pragma unroll
        for (int e = 0; e < kPer; e += 2)
            *reinterpret_cast<__nv_bfloat162*>(dst + e) = __floats2bfloat162_rn(acc[e] * inv, acc[e + 1] * inv);
        if (lse && lane == 0)
            lse[(size_t)hd * q_tokens + qi] =
                wsum > 0.f ? (lmax + log2f(wsum)) * 0.6931471805599453f : -INFINITY;
    }
}

__device__ int g_status = 0;
std::atomic<int> g_skip_loads{0};

// ------------------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

int make_cache_map(CUtensorMap* map, const void* base, int kv_tokens, int heads, int kD) {
    auto enc = get_encode();
    if (!enc) return vdit::fail(VDIT_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)kv_tokens, (cuuint64_t)heads};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)kv_tokens * kD * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kTile, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return vdit::fail(VDIT_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    return VDIT_OK;
}

// Per-device state of this file's kernels, set up once per device with that device current:
// the dynamic shared-memory opt-in of every attention kernel instance (a function attribute
// belongs to the function in one device's context), the device addresses of the status word and
// of the no-allocation scratch buffer (cudaGetSymbolAddress; in host code a __device__ variable's
// name is only a host-side stand-in), and the SM count. vdit_plan_upload runs this set-up for its
// device, so the forward calls on an uploaded plan find it done.
struct DeviceState {
    bool ready = false;
    int* status = nullptr;
    void* noalloc = nullptr;
    int sms = 148;
};
constexpr int kMaxDevices = 256;
std::mutex g_dev_mu;
DeviceState g_dev[kMaxDevices];

}  // namespace
// the no-allocation scratch buffer (its declaration and rules are with the entry point below)
static __device__ __align__(256) unsigned char g_noalloc_scratch[vdit::kNoAllocScratchBytes];
namespace {

int device_state(int dev, const DeviceState** out) {
    if (dev < 0 || dev >= kMaxDevices) return vdit::fail(VDIT_ERR_INVALID_ARG, "device index too large");
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceState& st = g_dev[dev];
    if (!st.ready) {
        const void* fns[4] = {(const void*)attn_fwd_kernel<128, false>, (const void*)attn_fwd_kernel<64, false>,
                              (const void*)attn_fwd_kernel<128, true>, (const void*)attn_fwd_kernel<64, true>};
        const int bytes[4] = {(int)Layout<128>::kSmemBytes, (int)Layout<64>::kSmemBytes,
                              (int)Layout<128>::kSmemBytes, (int)Layout<64>::kSmemBytes};
        for (int i = 0; i < 4; ++i)
            if (int rc = vdit::cuda_check(cudaFuncSetAttribute(fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                               bytes[i]),
                                          "cudaFuncSetAttribute(attention)"))
                return rc;
        void* p = nullptr;
        if (int rc = vdit::cuda_check(cudaGetSymbolAddress(&p, g_status), "cudaGetSymbolAddress(status)")) return rc;
        st.status = static_cast<int*>(p);
        p = nullptr;
        if (int rc = vdit::cuda_check(cudaGetSymbolAddress(&p, g_noalloc_scratch),
                                      "cudaGetSymbolAddress(no-alloc scratch)"))
            return rc;
        st.noalloc = p;
        if (int rc = vdit::cuda_check(cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev),
                                      "cudaDeviceGetAttribute"))
            return rc;
        st.ready = true;
    }
    *out = &st;
    return VDIT_OK;
}

// Tensor maps, arguments and launches of one forward pass (the attention kernel for the plan's
// head_dim and mode over the plan's CTA table, then the merge when the schedule cuts units into
// key pieces). ws_o / ws_lse: the pieces' scratch (unused when no unit is cut).
int launch_attention(const vdit_plan* p, const void* q, const void* k_cache, const void* v_cache,
                     void* o, float* lse, float scale, float* ws_o, float* ws_lse,
                     const vdit::RopeTables& tabs, cudaStream_t st, int dev, bool q_rotated = false) {
    using vdit::fail;
    CUtensorMap mk, mv;
    const int d = p->g.head_dim;
    if (int rc = make_cache_map(&mk, k_cache, p->kv_tokens, p->g.heads, d)) return rc;
    if (int rc = make_cache_map(&mv, v_cache, p->kv_tokens, p->g.heads, d)) return rc;
    const DeviceState* ds = nullptr;
    if (int rc = device_state(dev, &ds)) return rc;

    AttnArgs a{};
    a.u_row_ptr = p->d_u_row_ptr;
    a.u_col = p->d_u_col;
    a.u_flags = p->d_u_flags;
    a.cta = p->d_cta;
    a.cta_slot = p->d_cta_slot;
    a.ws_o = ws_o;
    a.ws_lse = ws_lse;
    a.masks = p->d_masks;
    a.u_mask = p->d_u_mask;
    a.q = static_cast<const uint4*>(q);
    a.o = static_cast<uint4*>(o);
    a.lse = lse;
    a.tt = static_cast<const float2*>(tabs.t);
    a.th = static_cast<const float2*>(tabs.h);
    a.tw = static_cast<const float2*>(tabs.w);
    a.status = ds->status;
    a.q_rotated = q_rotated ? 1 : 0;
    a.skip_loads = g_skip_loads.load(std::memory_order_relaxed);
    a.bt2 = p->g.band_t / 2;
    a.bh2 = p->g.band_h / 2;
    a.bw2 = p->g.band_w / 2;
    a.q_tokens = p->q_tokens;
    a.kv_tokens = p->kv_tokens;
    a.heads = p->g.heads;
    a.grid_h = p->g.grid_h;
    a.grid_w = p->g.grid_w;
    a.q_start = p->q_start;
    a.scale_log2 = (float)((double)scale * 1.4426950408889634);
    a.tau_log2 = (float)(p->m.tau * 1.4426950408889634);
    const bool dyn = p->m.kind & VDIT_MASK_DYNAMIC;
    const int n_cta = (int)(p->cta.size() / 5), n_cut = (int)(p->merge.size() / 4);
    if (n_cta == 0) return VDIT_OK;
    const dim3 grid((unsigned)n_cta);
    if (d == 128 && !dyn)
        attn_fwd_kernel<128, false><<<grid, kThreads, Layout<128>::kSmemBytes, st>>>(mk, mv, a);
    else if (d == 64 && !dyn)
        attn_fwd_kernel<64, false><<<grid, kThreads, Layout<64>::kSmemBytes, st>>>(mk, mv, a);
    else if (d == 128)
        attn_fwd_kernel<128, true><<<grid, kThreads, Layout<128>::kSmemBytes, st>>>(mk, mv, a);
    else
        attn_fwd_kernel<64, true><<<grid, kThreads, Layout<64>::kSmemBytes, st>>>(mk, mv, a);
    if (int rc = vdit::cuda_check(cudaGetLastError(), "attention kernel launch")) return rc;
    if (n_cut > 0) {
        const long long rows = (long long)n_cut * kQTiles * kTile;
        const int blocks = (int)std::min<long long>((rows + 7) / 8, (long long)ds->sms * 8);
        auto* ob = static_cast<__nv_bfloat16*>(o);
        const int4* mg = reinterpret_cast<const int4*>(p->d_merge);
        if (d == 128)
            split_combine_kernel<128><<<blocks, 256, 0, st>>>(ws_o, ws_lse, mg, n_cut, p->q_tokens,
                                                              p->g.heads, ob, lse);
        else
            split_combine_kernel<64><<<blocks, 256, 0, st>>>(ws_o, ws_lse, mg, n_cut, p->q_tokens,
                                                             p->g.heads, ob, lse);
        return vdit::cuda_check(cudaGetLastError(), "split merge launch");
    }
    return VDIT_OK;
}

}  // namespace

namespace {
int attn_forward_impl(const vdit_plan* p, const void* q, const void* k_cache, const void* v_cache, void* o,
                      float* lse, float scale, void* stream, bool q_rotated) {
    using vdit::fail;
    if (!p) return fail(VDIT_ERR_INVALID_ARG, "NULL plan");
    if (!p->d_buf) return fail(VDIT_ERR_NOT_UPLOADED, "plan not uploaded (vdit_plan_upload)");
    if (!q || !k_cache || !v_cache || !o) return fail(VDIT_ERR_INVALID_ARG, "NULL tensor");
    auto al = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15) == 0; };
    if (!al(q) || !al(k_cache) || !al(v_cache) || !al(o) || (reinterpret_cast<uintptr_t>(lse) & 3))
        return fail(VDIT_ERR_MISALIGNED, "tensor not aligned");
    if (!(scale > 0.f) || !std::isfinite(scale)) return fail(VDIT_ERR_INVALID_ARG, "scale must be > 0");
    int dev = 0;
    if (int rc = vdit::cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
    if (dev != p->device) return fail(VDIT_ERR_INVALID_ARG, "plan was uploaded to another device");
    vdit::RopeTables tabs;
    if (int rc = vdit::get_rope_tables(&p->g, &tabs)) return rc;
    return launch_attention(p, q, k_cache, v_cache, o, lse, scale, p->d_ws_o, p->d_ws_lse, tabs,
                            static_cast<cudaStream_t>(stream), dev, q_rotated);
}
}  // namespace

extern "C" int vdit_attn_forward(const vdit_plan* p, const void* q, const void* k_cache,
                                 const void* v_cache, void* o, float* lse, float scale,
                                 void* stream) {
    return attn_forward_impl(p, q, k_cache, v_cache, o, lse, scale, stream, false);
}

extern "C" int vdit_attn_forward_rotated(const vdit_plan* p, const void* q_rotated, const void* k_cache,
                                         const void* v_cache, void* o, float* lse, float scale,
                                         void* stream) {
    return attn_forward_impl(p, q_rotated, k_cache, v_cache, o, lse, scale, stream, true);
}

extern "C" void vdit_debug_skip_loads(int on) { g_skip_loads.store(on ? 1 : 0); }

extern "C" int vdit_get_status(int* status) {
    if (!status) return vdit::fail(VDIT_ERR_INVALID_ARG, "NULL status");
    if (int rc = vdit::cuda_check(cudaDeviceSynchronize(), "cudaDeviceSynchronize")) return rc;
    int zero = 0, v = 0;
    if (int rc = vdit::cuda_check(cudaMemcpyFromSymbol(&v, g_status, sizeof(int)), "read status"))
        return rc;
    if (int rc = vdit::cuda_check(cudaMemcpyToSymbol(g_status, &zero, sizeof(int)), "clear status"))
        return rc;
    int vq = 0;
    if (int rc = vdit::qkv_status_take(&vq)) return rc;
    *status = v != VDIT_OK ? v : vq;
    return VDIT_OK;
}

namespace vdit {
int attn_prepare_device(int dev) {
    const DeviceState* ds = nullptr;
    return device_state(dev, &ds);
}
}  // namespace vdit

// ------------------------------------------------------------------------------ no-allocation
// variant of the forward pass
//
// Some callers cannot call cudaMalloc at the moment they run attention: code that runs while
// another framework owns the device's memory through its own pool (a cudaMalloc there fails or
// fragments that pool), latency-critical loops that must not touch the allocator, and code that
// must not synchronise the device. vdit_attn_forward takes its key-split scratch from the plan
// (allocated by vdit_plan_upload); this variant instead writes the partial results into the
// fixed buffer g_noalloc_scratch, so the call itself allocates nothing.
//
// The buffer is a file-scope device array: every GPU on which this file's module is loaded holds
// its kNoAllocScratchBytes until the process exits. Under CUDA's lazy module loading the module
// (code and buffer) is loaded on first use on each device; vdit_plan_upload, which allocates
// anyway, makes that first use (it resolves the buffer's device address with
// cudaGetSymbolAddress, with the device current), so the variant itself, which needs an uploaded
// plan, only launches. All calls share the buffer and it keeps the last call's contents: every
// partial entry a successful call reads is written by the same call first, so nothing has to
// start at zero, but two calls whose kernels overlap on the GPU (different streams, same device)
// race on it. A call whose kernel timed out (VDIT_ERR_TIMEOUT from vdit_get_status) leaves o and
// lse unspecified: the merge may have read an earlier call's partials.
extern "C" int vdit_attn_forward_noalloc(const vdit_plan* p, const void* q, const void* k_cache,
                                         const void* v_cache, void* o, float* lse, float scale,
                                         void* stream) {
    using vdit::fail;
    if (!p) return fail(VDIT_ERR_INVALID_ARG, "NULL plan");
    if (!p->d_buf) return fail(VDIT_ERR_NOT_UPLOADED, "plan not uploaded (vdit_plan_upload)");
    if (!q || !k_cache || !v_cache || !o) return fail(VDIT_ERR_INVALID_ARG, "NULL tensor");
    auto al = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15) == 0; };
    if (!al(q) || !al(k_cache) || !al(v_cache) || !al(o) || (reinterpret_cast<uintptr_t>(lse) & 3))
        return fail(VDIT_ERR_MISALIGNED, "tensor not aligned");
    if (!(scale > 0.f) || !std::isfinite(scale)) return fail(VDIT_ERR_INVALID_ARG, "scale must be > 0");
    int dev = 0;
    if (int rc = vdit::cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
    if (dev != p->device) return fail(VDIT_ERR_INVALID_ARG, "plan was uploaded to another device");
    // scratch this plan's key pieces need: partial O [slot][256][d] fp32, then partial
    // log2-sum-exp [slot][256] fp32 (the schedule keeps the slots within the buffer)
    const int d = p->g.head_dim;
    const size_t o_bytes = sizeof(float) * (size_t)p->n_slots * kQTiles * kTile * d;
    const size_t l_bytes = sizeof(float) * (size_t)p->n_slots * kQTiles * kTile;
    if (o_bytes + l_bytes > vdit::kNoAllocScratchBytes)
        return fail(VDIT_ERR_UNSUPPORTED,
                    "internal: this plan's key pieces need " + std::to_string(o_bytes + l_bytes) +
                        " bytes of scratch; the no-allocation buffer holds " +
                        std::to_string(vdit::kNoAllocScratchBytes));
    const DeviceState* ds = nullptr;
    if (int rc = device_state(dev, &ds)) return rc;
    void* scratch = ds->noalloc;
    vdit::RopeTables tabs;
    if (int rc = vdit::find_rope_tables(&p->g, &tabs)) return rc;
    float* ws_o = p->n_slots ? static_cast<float*>(scratch) : nullptr;
    float* ws_lse = p->n_slots ? reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + o_bytes)
                               : nullptr;
    return launch_attention(p, q, k_cache, v_cache, o, lse, scale, ws_o, ws_lse, tabs,
                            static_cast<cudaStream_t>(stream), dev);
}
