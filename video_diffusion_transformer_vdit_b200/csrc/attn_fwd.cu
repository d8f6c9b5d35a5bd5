// Masked spatio-temporal attention forward on tcgen05 tensor cores (libvdit, sm_100a).
//
// Computes o = softmax(R(p_q) q . R(p_k) k * scale, restricted to the mask) v for every
// (query tile, head) of a plan: the O(N^2) step of full spatio-temporal attention ("Accelerating
// Video Generation Inference with Sequential-Parallel 3D Positional Encoding Using a Global Time
// Index", section 1) over the block-causal / radial tile schedule ("DynamicRad", section 2;
// Wave Forcing / WaveRT block-causal chunks). Only the tiles the plan lists are visited; a tile
// flagged full skips the per-pair predicate.
//
// One CTA = one 128-row query tile of one head; 8 warps:
//   warp 0      producer: TMA (cp.async.bulk.tensor, SWIZZLE_128B) of the K and V tiles from the
//               head-major cache into a 2-stage ring, and the key-position table of partial tiles;
//   warp 1      TMEM allocator and MMA issuer (one thread): S = Q K^T into TMEM columns [0,128),
//               O += P V into columns [128,256), kind::f16 bf16 x bf16 -> fp32, M = N = 128;
//   warps 2-3   help stage Q, then idle;
//   warps 4-7   softmax: thread r owns query row r (TMEM lane r): tcgen05.ld of its S row, mask,
//               online softmax in fp32 (log2 domain, lazy rescale of O only when the running max
//               grows by more than 2^8), P as bf16 into shared memory (K-major, 128B swizzle) for
//               the PV MMA, epilogue (O / l -> bf16, staged through shared memory so the global
//               stores are 256-byte coalesced rows; natural-log LSE).
// Q is read from global memory, rotated (3-D RoPE at the plan's query positions, fp32 math on
// fp64-built tables) and written straight into the swizzled K-major layout the MMA reads: the
// RoPE of Q is fused into the Q load.
//
// Every mbarrier wait is bounded (globaltimer): on expiry the thread raises the CTA abort flag
// and the device status word (VDIT_ERR_TIMEOUT), every role leaves its loop, in-flight TMA and
// MMA work is drained (again bounded) and TMEM is freed before the CTA exits.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"

namespace {

constexpr int kTile = 128;
constexpr int kStages = 2;
constexpr int kThreads = 256;
constexpr uint32_t kSlabBytes = kTile * 64 * 2;  // 16 KiB: 128 rows x 128 B (one swizzle width)
constexpr uint32_t kPBytes = kTile * kTile * 2;  // P tile: 128 queries x 128 keys, bf16
constexpr uint32_t kTmemCols = 256;              // S: columns [0,128), O: [128, 128 + D)
constexpr float kRescaleTau = 8.0f;              // rescale O only when the max grows by > 2^8
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// barrier indices (8 bytes each)
enum {
    B_KFULL = 0, B_KEMPTY = B_KFULL + kStages, B_VFULL = B_KEMPTY + kStages,
    B_VEMPTY = B_VFULL + kStages, B_IFULL = B_VEMPTY + kStages, B_IEMPTY = B_IFULL + kStages,
    B_SFULL = B_IEMPTY + kStages, B_SFREE, B_PFULL, B_ODONE, B_DRAIN, B_COUNT
};
static_assert(B_COUNT <= 32, "barrier area too small");
constexpr uint32_t kKinfoBytes = 16 + kTile * 16;  // header (tile, full) + 128 x int4

// Shared-memory map for head_dim D (offsets from a 1024-byte aligned base).
template <int D>
struct Layout {
    static constexpr int kSlabs = D / 64;
    static constexpr uint32_t kTileBytes = kTile * D * 2;  // one Q, K or V tile
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = OFF_Q + kTileBytes;
    static constexpr uint32_t OFF_V = OFF_K + kStages * kTileBytes;
    static constexpr uint32_t OFF_P = OFF_V + kStages * kTileBytes;
    static constexpr uint32_t OFF_BAR = OFF_P + kPBytes;
    static constexpr uint32_t OFF_MISC = OFF_BAR + 8 * 32;  // [0] tmem base, [1] abort flag
    static constexpr uint32_t OFF_KINFO = OFF_MISC + 64;
    static constexpr uint32_t OFF_RAD = OFF_KINFO + kStages * kKinfoBytes;
    static constexpr uint32_t kSmemBytes = OFF_RAD + (VDIT_MAX_DT + 1) * 4 + 1024;  // + align slack
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
    static_assert(kTile * D * 2 <= kPBytes, "O staging must fit in the P buffer");
};

struct AttnArgs {
    const int* row_ptr;
    const int* col_idx;
    const unsigned char* full;
    const int* slot_frame;
    const int* radius;
    const uint4* q;
    uint4* o;
    float* lse;
    const float2* tt;
    const float2* th;
    const float2* tw;
    int* status;
    int bt2, bh2, bw2;
    int q_tokens, kv_tokens, heads;
    int grid_h, grid_w;
    int q_start;
    int causal, chunk_frames;
    int dt_max;
    float scale_log2;
};

// ------------------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Waits for the phase of `bar` with the given parity. Gives up (returns false) after
// kWaitLimitNs, or as soon as another thread of the CTA has given up.
__device__ __noinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 15) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                atomicExch(status, VDIT_ERR_TIMEOUT);
                return false;
            }
        }
    }
}
// Warp-uniform form: every lane waits, and the warp continues only if all lanes succeeded, so
// a timeout never leaves part of a warp inside a .sync.aligned sequence.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* status) {
    const bool ok = wait_bounded(bar, parity, abort_flag, status);
    return __all_sync(0xffffffffu, ok);
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

#define VDIT_R32(r, i) "=r"(r[i + 0]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
    "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define VDIT_W32(r, i) "r"(r[i + 0]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
    "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])
#define VDIT_RW32(r, i) "+r"(r[i + 0]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), \
    "+r"(r[i + 4]), "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7])

// 32 consecutive fp32 columns of this thread's TMEM lane (warp-collective, asynchronous).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : VDIT_R32(r, 0), VDIT_R32(r, 8), VDIT_R32(r, 16), VDIT_R32(r, 24)
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        VDIT_W32(r, 0), VDIT_W32(r, 8), VDIT_W32(r, 16), VDIT_W32(r, 24)
        : "memory");
}
// Waits for this thread's outstanding tcgen05.ld and ties the 32 registers to the wait, so no
// use of them can be scheduled before it.
__device__ __forceinline__ void tmem_ld_wait(uint32_t* r) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : VDIT_RW32(r, 0), VDIT_RW32(r, 8), VDIT_RW32(r, 16), VDIT_RW32(r, 24)
                 :
                 : "memory");
}
__device__ __forceinline__ void reg_touch32(uint32_t* r) {
    asm volatile("" : VDIT_RW32(r, 0), VDIT_RW32(r, 8), VDIT_RW32(r, 16), VDIT_RW32(r, 24));
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 format (version 1 at bit 46).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo_bytes >> 4) << 16) |
           ((uint64_t)(sbo_bytes >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulate, M = 128, N = n, A K-major,
// B K-major (b_mn = 0) or MN-major (b_mn = 1).
__host__ __device__ constexpr uint32_t instr_desc(uint32_t n, uint32_t b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn << 16) | ((n >> 3) << 17) |
           ((uint32_t)(kTile >> 4) << 24);
}

// Byte offset of 16-byte chunk c16 (channels 8*c16 .. 8*c16+7) of row r in a 128 x 128 bf16
// tile stored K-major with the 128-byte swizzle: two 64-channel slabs of 128 rows x 128 bytes,
// chunk j of row r at position j ^ (r mod 8).
__device__ __forceinline__ uint32_t sw128_offset(int r, int c16) {
    return (uint32_t)((c16 >> 3) * kSlabBytes + r * 128 + (((c16 & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint4 rope_chunk(uint4 in, int pp0, int t, int h, int w,
                                            const AttnArgs& a) {
    uint32_t word[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int pp = pp0 + i;
        float2 cs;
        if (pp < a.bt2)
            cs = __ldg(a.tt + (size_t)t * a.bt2 + pp);
        else if (pp < a.bt2 + a.bh2)
            cs = __ldg(a.th + h * a.bh2 + (pp - a.bt2));
        else
            cs = __ldg(a.tw + w * a.bw2 + (pp - a.bt2 - a.bh2));
        __nv_bfloat162 b;
        memcpy(&b, &word[i], 4);
        const float2 x = __bfloat1622float2(b);
        b = __floats2bfloat162_rn(fmaf(x.x, cs.x, -x.y * cs.y), fmaf(x.x, cs.y, x.y * cs.x));
        memcpy(&word[i], &b, 4);
    }
    return make_uint4(word[0], word[1], word[2], word[3]);
}

// ------------------------------------------------------------------------------ the kernel

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const AttnArgs a) {
    using L = Layout<D>;
    constexpr uint32_t kTileBytes = L::kTileBytes;
    constexpr uint32_t OFF_Q = L::OFF_Q, OFF_K = L::OFF_K, OFF_V = L::OFF_V, OFF_P = L::OFF_P;
    constexpr uint32_t OFF_BAR = L::OFF_BAR, OFF_MISC = L::OFF_MISC, OFF_KINFO = L::OFF_KINFO;
    constexpr uint32_t OFF_RAD = L::OFF_RAD;
    constexpr int kC16 = D / 8;  // 16-byte chunks per head row
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + OFF_BAR;
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
    int* rad_s = reinterpret_cast<int*>(smem + OFF_RAD);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qt = blockIdx.x, head = blockIdx.y;
    const int t_begin = __ldg(a.row_ptr + qt);
    const int n_tiles = __ldg(a.row_ptr + qt + 1) - t_begin;
    const int ft = a.grid_h * a.grid_w;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(BAR(B_KFULL + s), 1);
            mbar_init(BAR(B_KEMPTY + s), 1);
            mbar_init(BAR(B_VFULL + s), 1);
            mbar_init(BAR(B_VEMPTY + s), 1);
            mbar_init(BAR(B_IFULL + s), 1);
            mbar_init(BAR(B_IEMPTY + s), 128);
        }
        mbar_init(BAR(B_SFULL), 1);
        mbar_init(BAR(B_SFREE), 128);
        mbar_init(BAR(B_PFULL), 128);
        mbar_init(BAR(B_ODONE), 1);
        mbar_init(BAR(B_DRAIN), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         sbase + OFF_MISC),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // radius table and the rotated Q tile (all 256 threads)
    for (int i = threadIdx.x; i <= a.dt_max; i += kThreads) rad_s[i] = __ldg(a.radius + i);
    {
        const int q0 = qt * kTile;
#pragma unroll 2
        for (int i = 0; i < (kTile * kC16) / kThreads; ++i) {
            const int idx = threadIdx.x + i * kThreads;
            const int r = idx / kC16, c16 = idx % kC16;
            const int qi = q0 + r;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (qi < a.q_tokens) {
                const int f = qi / ft, rem = qi - f * ft;
                const int hh = rem / a.grid_w, ww = rem - hh * a.grid_w;
                const uint4 x = __ldg(a.q + ((size_t)qi * a.heads + head) * kC16 + c16);
                v = rope_chunk(x, c16 * 4, a.q_start + f, hh, ww, a);
            }
            *reinterpret_cast<uint4*>(smem + OFF_Q + sw128_offset(r, c16)) = v;
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const uint32_t tmem_s = tmem, tmem_o = tmem + 128;

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        int issued = 0;
        for (int it = 0; it < n_tiles; ++it) {
            const int s = it % kStages;
            const uint32_t ph = (uint32_t)((it / kStages) - 1) & 1u;
            const int kt = __ldg(a.col_idx + t_begin + it);
            const int full = __ldg(a.full + t_begin + it);
            if (it >= kStages && !warp_wait(BAR(B_KEMPTY + s), ph, abort_flag, a.status)) break;
            if (lane == 0) {
                mbar_expect_tx(BAR(B_KFULL + s), kTileBytes);
                const uint32_t dst = sbase + OFF_K + s * kTileBytes;
#pragma unroll
                for (int sl = 0; sl < L::kSlabs; ++sl)
                    tma_load_3d(dst + sl * kSlabBytes, &tmap_k, BAR(B_KFULL + s), 64 * sl, kt * kTile, head);
            }
            // key positions of a partial tile (one int4 per key: frame, h, w, causal chunk)
            if (it >= kStages && !warp_wait(BAR(B_IEMPTY + s), ph, abort_flag, a.status)) {
                issued = it * 2 + 1;
                break;
            }
            uint8_t* info = smem + OFF_KINFO + s * kKinfoBytes;
            if (lane == 0) {
                reinterpret_cast<int*>(info)[0] = kt;
                reinterpret_cast<int*>(info)[1] = full;
            }
            if (!full) {
                int4* ki = reinterpret_cast<int4*>(info + 16);
                for (int j = lane; j < kTile; j += 32) {
                    const int key = kt * kTile + j;
                    int4 e = make_int4(-1, 0, 0, 0x7fffffff);
                    if (key < a.kv_tokens) {
                        const int slot = key / ft, rem = key - slot * ft;
                        const int hh = rem / a.grid_w;
                        const int tk = __ldg(a.slot_frame + slot);
                        e = make_int4(tk, hh, rem - hh * a.grid_w,
                                      (tk >= 0 && a.causal) ? tk / a.chunk_frames : 0);
                        if (tk < 0) e.w = 0x7fffffff;
                    }
                    ki[j] = e;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(B_IFULL + s));
            if (it >= kStages && !warp_wait(BAR(B_VEMPTY + s), ph, abort_flag, a.status)) {
                issued = it * 2 + 1;
                break;
            }
            if (lane == 0) {
                mbar_expect_tx(BAR(B_VFULL + s), kTileBytes);
                const uint32_t dst = sbase + OFF_V + s * kTileBytes;
#pragma unroll
                for (int sl = 0; sl < L::kSlabs; ++sl)
                    tma_load_3d(dst + sl * kSlabBytes, &tmap_v, BAR(B_VFULL + s), 64 * sl, kt * kTile, head);
            }
            issued = it * 2 + 2;
            __syncwarp();
        }
        // drain: every TMA this warp issued must have landed before the CTA may exit
        if (*abort_flag) {
            for (int j = (issued - 2 * kStages > 0 ? issued - 2 * kStages : 0); j < issued; ++j) {
                const int it = j >> 1, s = it % kStages;
                const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                const int b = (j & 1) ? B_VFULL + s : B_KFULL + s;
                // a landed load completes the phase; give up only on the time limit
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(BAR(b), ph) && globaltimer() - t0 < kWaitLimitNs) {
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_tiles > 0) {
            constexpr uint32_t idesc_qk = instr_desc(kTile, 0), idesc_pv = instr_desc(D, 1);
            const uint32_t q_addr = sbase + OFF_Q, p_addr = sbase + OFF_P;
            auto issue_qk = [&](int s) {
                const uint32_t k_addr = sbase + OFF_K + s * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kSlabBytes + (kk & 3) * 32;
                    tc_mma(tmem_s, smem_desc_sw128(q_addr + off, 16, 1024),
                           smem_desc_sw128(k_addr + off, 16, 1024), idesc_qk, kk > 0);
                }
            };
            bool ok = wait_bounded(BAR(B_KFULL + 0), 0, abort_flag, a.status);
            if (ok) {
                tc_fence_after();
                issue_qk(0);
                tc_commit(BAR(B_SFULL));
                tc_commit(BAR(B_KEMPTY + 0));
            }
            for (int it = 0; ok && it < n_tiles; ++it) {
                const int s = it % kStages;
                if (it + 1 < n_tiles) {
                    const int s1 = (it + 1) % kStages;
                    if (!wait_bounded(BAR(B_KFULL + s1), ((it + 1) / kStages) & 1, abort_flag, a.status) ||
                        !wait_bounded(BAR(B_SFREE), it & 1, abort_flag, a.status))
                        break;
                    tc_fence_after();
                    issue_qk(s1);
                    tc_commit(BAR(B_SFULL));
                    tc_commit(BAR(B_KEMPTY + s1));
                }
                if (!wait_bounded(BAR(B_PFULL), it & 1, abort_flag, a.status) ||
                    !wait_bounded(BAR(B_VFULL + s), (it / kStages) & 1, abort_flag, a.status))
                    break;
                tc_fence_after();
                const uint32_t v_addr = sbase + OFF_V + s * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    const uint32_t poff = (kk >> 2) * kSlabBytes + (kk & 3) * 32;
                    tc_mma(tmem_o, smem_desc_sw128(p_addr + poff, 16, 1024),
                           smem_desc_sw128(v_addr + kk * 16 * 128, kSlabBytes, 1024), idesc_pv,
                           (it > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(BAR(B_ODONE));
                tc_commit(BAR(B_VEMPTY + s));
            }
        }
        if (lane == 0) {
            // drain: all MMAs issued by this thread complete before TMEM is released
            tc_commit(BAR(B_DRAIN));
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(BAR(B_DRAIN), 0) && globaltimer() - t0 < kWaitLimitNs) {
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------------ softmax
        const int row = threadIdx.x - 128;  // TMEM lane == query row within the tile
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const int qi = qt * kTile + row;
        const int qf = qi / ft, qrem = qi - qf * ft;
        const int tq = a.q_start + qf, hq = qrem / a.grid_w, wq = qrem - (qrem / a.grid_w) * a.grid_w;
        const int cq = a.causal ? tq / a.chunk_frames : 0x7fffffff;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int it = 0; it < n_tiles; ++it) {
            const int s = it % kStages;
            if (!warp_wait(BAR(B_SFULL), it & 1, abort_flag, a.status)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tmem_s + lane_base + c * 32, sr + c * 32);
            tmem_ld_wait(sr);
            reg_touch32(sr + 32);
            reg_touch32(sr + 64);
            reg_touch32(sr + 96);
            tc_fence_before();
            mbar_arrive(BAR(B_SFREE));
            float sv[128];
#pragma unroll
            for (int j = 0; j < 128; ++j) sv[j] = __uint_as_float(sr[j]) * a.scale_log2;

            if (!warp_wait(BAR(B_IFULL + s), (it / kStages) & 1, abort_flag, a.status)) { ok = false; break; }
            const uint8_t* info = smem + OFF_KINFO + s * kKinfoBytes;
            const int full = reinterpret_cast<const int*>(info)[1];
            if (!full) {
                const int4* ki = reinterpret_cast<const int4*>(info + 16);
#pragma unroll
                for (int j = 0; j < 128; ++j) {
                    const int4 e = ki[j];
                    int dt = abs(tq - e.x);
                    dt = dt > a.dt_max ? a.dt_max : dt;
                    const int cheb = max(abs(hq - e.y), abs(wq - e.z));
                    const bool keep = (e.x >= 0) & (e.w <= cq) & (cheb <= rad_s[dt]);
                    sv[j] = keep ? sv[j] : -INFINITY;
                }
            }
            mbar_arrive(BAR(B_IEMPTY + s));

            float mx = sv[0];
#pragma unroll
            for (int j = 1; j < 128; ++j) mx = fmaxf(mx, sv[j]);
            const float m_new = fmaxf(m, mx);
            const bool resc = m_new > m + kRescaleTau;
            float alpha = 1.f;
            if (resc) {
                alpha = fast_exp2(m - m_new);
                m = m_new;
            }
            const float m_use = (m == -INFINITY) ? 0.f : m;
            float rs = 0.f;
            uint32_t pk[64];
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                const float p0 = fast_exp2(sv[2 * j] - m_use), p1 = fast_exp2(sv[2 * j + 1] - m_use);
                rs += p0 + p1;
                __nv_bfloat162 b = __floats2bfloat162_rn(p0, p1);
                memcpy(&pk[j], &b, 4);
            }
            l = l * alpha + rs;

            // PV of the previous tile must be done before O is rescaled or P is overwritten
            if (it > 0) {
                if (!warp_wait(BAR(B_ODONE), (it - 1) & 1, abort_flag, a.status)) { ok = false; break; }
                tc_fence_after();
                if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t orow[32];
                        tmem_ld32(tmem_o + lane_base + c * 32, orow);
                        tmem_ld_wait(orow);
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            orow[j] = __float_as_uint(__uint_as_float(orow[j]) * alpha);
                        tmem_st32(tmem_o + lane_base + c * 32, orow);
                    }
                    tmem_st_wait();
                }
            }
#pragma unroll
            for (int c16 = 0; c16 < 16; ++c16)
                *reinterpret_cast<uint4*>(smem + OFF_P + sw128_offset(row, c16)) =
                    make_uint4(pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2], pk[4 * c16 + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(BAR(B_PFULL));
        }
        if (ok && n_tiles > 0) {
            if (!warp_wait(BAR(B_ODONE), (n_tiles - 1) & 1, abort_flag, a.status)) ok = false;
        }
        // every softmax thread reaches this barrier (aborted or not); any failure skips the
        // epilogue for the whole warpgroup
        int any_fail;
        asm volatile(
            "{\n\t.reg .pred p, q;\n\t"
            "setp.eq.u32 p, %1, 0;\n\t"
            "bar.red.or.pred q, 1, 128, p;\n\t"
            "selp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(any_fail)
            : "r"((uint32_t)ok)
            : "memory");
        if (!any_fail) {
            tc_fence_after();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            uint8_t* stage = smem + OFF_P;  // P is no longer needed: stage O rows here
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t orow[32];
                if (n_tiles > 0) {
                    tmem_ld32(tmem_o + lane_base + c * 32, orow);
                    tmem_ld_wait(orow);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) orow[j] = 0u;
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t wds[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat162 b = __floats2bfloat162_rn(
                            __uint_as_float(orow[q4 * 8 + 2 * e]) * inv_l,
                            __uint_as_float(orow[q4 * 8 + 2 * e + 1]) * inv_l);
                        memcpy(&wds[e], &b, 4);
                    }
                    const int chunk = c * 4 + q4;
                    *reinterpret_cast<uint4*>(stage + row * (D * 2) + ((chunk ^ (row & 7)) << 4)) =
                        make_uint4(wds[0], wds[1], wds[2], wds[3]);
                }
            }
            if (a.lse && qi < a.q_tokens)
                a.lse[(size_t)head * a.q_tokens + qi] =
                    l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
            asm volatile("bar.sync 2, 128;" ::: "memory");
            const int t = threadIdx.x - 128;
#pragma unroll 4
            for (int i = 0; i < kC16; ++i) {
                const int r = i * (128 / kC16) + t / kC16, chunk = t % kC16;
                const int qr = qt * kTile + r;
                if (qr < a.q_tokens) {
                    const uint4 v = *reinterpret_cast<const uint4*>(stage + r * (D * 2) + ((chunk ^ (r & 7)) << 4));
                    __stcs(a.o + ((size_t)qr * a.heads + head) * kC16 + chunk, v);
                }
            }
        }
    }
    // ---------------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
    }
}

__device__ int g_status = 0;

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

int* status_ptr() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    return static_cast<int*>(p);
}

}  // namespace

extern "C" int vdit_attn_forward(const vdit_plan* p, const void* q, const void* k_cache,
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
    vdit::RopeTables tabs;
    if (int rc = vdit::get_rope_tables(&p->g, &tabs)) return rc;
    CUtensorMap mk, mv;
    const int d = p->g.head_dim;
    if (int rc = make_cache_map(&mk, k_cache, p->kv_tokens, p->g.heads, d)) return rc;
    if (int rc = make_cache_map(&mv, v_cache, p->kv_tokens, p->g.heads, d)) return rc;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(attn_fwd_kernel<128>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)Layout<128>::kSmemBytes);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(attn_fwd_kernel<64>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)Layout<64>::kSmemBytes);
    });
    if (int rc = vdit::cuda_check(attr_err, "cudaFuncSetAttribute")) return rc;
    int* status = status_ptr();
    if (!status) return fail(VDIT_ERR_CUDA, "cannot resolve status word");

    AttnArgs a{};
    a.row_ptr = p->d_row_ptr;
    a.col_idx = p->d_col_idx;
    a.full = p->d_full;
    a.slot_frame = p->d_slot_frame;
    a.radius = p->d_radius;
    a.q = static_cast<const uint4*>(q);
    a.o = static_cast<uint4*>(o);
    a.lse = lse;
    a.tt = static_cast<const float2*>(tabs.t);
    a.th = static_cast<const float2*>(tabs.h);
    a.tw = static_cast<const float2*>(tabs.w);
    a.status = status;
    a.bt2 = p->g.band_t / 2;
    a.bh2 = p->g.band_h / 2;
    a.bw2 = p->g.band_w / 2;
    a.q_tokens = p->q_tokens;
    a.kv_tokens = p->kv_tokens;
    a.heads = p->g.heads;
    a.grid_h = p->g.grid_h;
    a.grid_w = p->g.grid_w;
    a.q_start = p->q_start;
    a.causal = (p->m.kind & VDIT_MASK_BLOCK_CAUSAL) ? 1 : 0;
    a.chunk_frames = a.causal ? p->m.chunk_frames : 1;
    a.dt_max = p->dt_max;
    a.scale_log2 = (float)((double)scale * 1.4426950408889634);
    dim3 grid(p->n_qt, p->g.heads);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d == 128)
        attn_fwd_kernel<128><<<grid, kThreads, Layout<128>::kSmemBytes, st>>>(mk, mv, a);
    else
        attn_fwd_kernel<64><<<grid, kThreads, Layout<64>::kSmemBytes, st>>>(mk, mv, a);
    return vdit::cuda_check(cudaGetLastError(), "attention kernel launch");
}

extern "C" int vdit_get_status(int* status) {
    if (!status) return vdit::fail(VDIT_ERR_INVALID_ARG, "NULL status");
    if (int rc = vdit::cuda_check(cudaDeviceSynchronize(), "cudaDeviceSynchronize")) return rc;
    int zero = 0, v = 0;
    if (int rc = vdit::cuda_check(cudaMemcpyFromSymbol(&v, g_status, sizeof(int)), "read status"))
        return rc;
    if (int rc = vdit::cuda_check(cudaMemcpyToSymbol(g_status, &zero, sizeof(int)), "clear status"))
        return rc;
    *status = v;
    return VDIT_OK;
}
