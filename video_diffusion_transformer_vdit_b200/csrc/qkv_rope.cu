// Fused QKV projection + 3-D RoPE + KV-cache append on tcgen05 tensor cores (libvdit, sm_100a).
//
// "Accelerating Video Generation Inference with Sequential-Parallel 3D Positional Encoding Using
// a Global Time Index", section 2.C, fuses the QKV projections and the causal RoPE into one
// kernel; section 2.B gives each chunk global temporal positions t = start_frame + local frame;
// section 2.A keeps K and V of past chunks in a cache. Here one persistent GEMM computes
//   [Q | K | V] = X W^T        (X [tokens, d_model], W [3 * heads * head_dim, d_model], bf16)
// in fp32 on the tensor cores and its epilogue rotates Q and K at the tokens' global positions
// (fp32 math, tables built in fp64) and stores bf16: Q to [tokens, heads, head_dim], K' and V
// straight into the chunk's frame slots of the head-major ring cache (what vdit_kv_append does).
//
// Pairs of CTAs (clusters of two, one CTA per SM) run persistent over 256 x 256 output tiles (in
// the order that keeps the smaller operand in L2) with tcgen05 cta_group::2: one M = 256, N = 256,
// K = 16 MMA covers the tile, CTA r of the pair staging the X rows m0 + 128 r .. and the W rows
// n0 + 128 r .. of each 64-wide k step, and receiving its 128 output rows in its own TMEM. 6 warps
// per CTA:
//   warp 0      producer: TMA (SWIZZLE_128B) of the CTA's 128 x 64 X and W tiles into a 5-stage
//               ring; both CTAs' copies complete on the first CTA's stage barrier;
//   warp 1      paired TMEM allocation (512 columns in each CTA: two 256-column fp32
//               accumulators); in the first CTA, the single thread issuing the MMAs (four per k
//               step), which commits them to the barriers of both CTAs;
//   warps 2-5   epilogue of the CTA's 128 rows: thread r owns accumulator row r (TMEM lane r);
//               per 64-column slab it loads the fp32 row (tcgen05.ld), rotates the pairs, rounds
//               to bf16 into a swizzled shared-memory slab and one thread stores the slab with a
//               TMA tensor store. The accumulator is released (on the first CTA's barrier, which
//               counts both CTAs' threads) as soon as it has been read, so the next tile's MMAs
//               overlap the stores.
// Per SM each MMA reads 8 KiB of operands in 128 cycles and TMA writes 32 KiB per k step: 128 B of
// shared-memory traffic per cycle at the tensor rate, where a single CTA's M = 128, N = 256 tile
// would need 192 (its B operand, 256 W rows, read whole by each CTA).
// Every mbarrier wait is bounded (globaltimer); on expiry the CTA raises its abort flag and the
// status word (VDIT_ERR_TIMEOUT), drains what it issued and frees TMEM before exiting.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sm100.h"

namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kGThreads = 192;
constexpr int kGWarpTMA = 0, kGWarpMMA = 1;  // warps 2-5: epilogue
constexpr uint32_t kOutSlab = kBM * 64 * 2;        // 16 KiB: 128 rows x 64 columns of bf16
constexpr uint32_t kAccCols = kBN;                 // fp32 columns per accumulator

struct GemmArgs {
    int m;              // tokens of this launch
    int k;              // d_model
    int n_tiles_m, n_tiles_n;  // 256 x 256 output tiles (a CTA pair each)
    int n_major;        // tile order: 0 = row blocks outer (W stays in L2), 1 = column blocks outer
    int hd;             // heads * head_dim (one of the Q, K, V sections)
    int head_dim;
    int tok0;           // chunk-local index of this launch's first token
    int start_frame;    // global frame of the chunk's first token
    int grid_h, grid_w;
    const float2* tt;
    const float2* th;
    const float2* tw;
    int bt2, bh2, bw2;
    int* status;
};

__device__ int g_qkv_status = 0;

// (cos, sin) of RoPE pair pp of a head vector at position (t, h, w): bands t, h, w in order.
__device__ __forceinline__ float2 pair_angle(int pp, int t, int h, int w, const GemmArgs& a) {
    const bool in_h = pp >= a.bt2, in_w = pp >= a.bt2 + a.bh2;
    const float2* tab = in_w ? a.tw : (in_h ? a.th : a.tt);
    const int row = in_w ? w : (in_h ? h : t);
    const int width = in_w ? a.bw2 : (in_h ? a.bh2 : a.bt2);
    const int jj = pp - (in_w ? a.bt2 + a.bh2 : (in_h ? a.bt2 : 0));
    return __ldg(tab + (size_t)row * width + jj);
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(map),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until at most n committed bulk groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ------------------------------------------------------------------------------ the kernel
constexpr int kPStages = 5;  // 4 / 5 / 6 stages measured 1 424 / 1 424 / 1 433 TFLOP/s (1.3B clip)
constexpr uint32_t kPABytes = 128 * kBK * 2;                      // 16 KiB of X rows
constexpr uint32_t kPBBytes = 128 * kBK * 2;                      // 16 KiB of W rows
constexpr uint32_t kPStageBytes = kPABytes + kPBBytes;
enum { PG_FULL = 0, PG_EMPTY = PG_FULL + kPStages, PG_AFULL = PG_EMPTY + kPStages,
       PG_AEMPTY = PG_AFULL + 2, PG_DRAIN = PG_AEMPTY + 2, PG_COUNT };
static_assert(PG_COUNT <= 32, "barrier area");
constexpr uint32_t OFF_PSTAGE = 0;
constexpr uint32_t OFF_POUT = OFF_PSTAGE + kPStages * kPStageBytes;
constexpr uint32_t OFF_PBAR = OFF_POUT + 2 * kOutSlab;
constexpr uint32_t OFF_PMISC = OFF_PBAR + 8 * 32;
constexpr uint32_t kPSmemBytes = OFF_PMISC + 64 + 1024;
static_assert(kPSmemBytes <= 227 * 1024, "shared memory budget");

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA load into this CTA's shared memory, completing on an mbarrier of either CTA of the pair.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(map), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives on the barrier at this offset in both CTAs of the pair once the MMAs issued so far
// have completed.
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"((unsigned short)3)
        : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGThreads, 1)
    qkv_rope_pair_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                         const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                         const __grid_constant__ CUtensorMap map_v, const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    auto BAR = [&](int i) { return sbase + OFF_PBAR + 8u * (uint32_t)i; };
    volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + OFF_PMISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_PMISC + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs; 1: its peer
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int n_tiles = a.n_tiles_m * a.n_tiles_n;  // 256 x 256 tiles
    const int k_steps = (a.k + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(BAR(PG_FULL + s), 1);
            mbar_init(BAR(PG_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(PG_AFULL + b), 1);
            mbar_init(BAR(PG_AEMPTY + b), 256);  // the epilogue threads of both CTAs
        }
        mbar_init(BAR(PG_DRAIN), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kGWarpMMA) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sbase + OFF_PMISC),
                     "r"(2 * kAccCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers are initialised before either signals the other's
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp == kGWarpTMA) {
        // ---------------------------------------------------------------------- producer
        int it = 0, issued = 0;
        bool ok = true;
        const uint32_t full0 = mapa_shared(BAR(PG_FULL), 0);  // the first CTA's stage barriers
        for (int tile = pair; ok && tile < n_tiles; tile += n_pairs) {
            int m0, n0;
            if (a.n_major) {
                m0 = (tile % a.n_tiles_m) * 256;
                n0 = (tile / a.n_tiles_m) * 256;
            } else {
                m0 = (tile / a.n_tiles_n) * 256;
                n0 = (tile % a.n_tiles_n) * 256;
            }
            for (int ks = 0; ks < k_steps; ++ks, ++it) {
                const int s = it % kPStages;
                if (it >= kPStages &&
                    !warp_wait(BAR(PG_EMPTY + s), (uint32_t)((it / kPStages) - 1) & 1u, abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    if (rank == 0) mbar_expect_tx(BAR(PG_FULL + s), 2 * kPStageBytes);
                    const uint32_t dst = sbase + OFF_PSTAGE + s * kPStageBytes;
                    tma_load_2d_pair(dst, &map_x, full0 + 8u * (uint32_t)s, ks * kBK, m0 + 128 * (int)rank);
                    tma_load_2d_pair(dst + kPABytes, &map_w, full0 + 8u * (uint32_t)s, ks * kBK, n0 + 128 * (int)rank);
                }
                issued = it + 1;
                __syncwarp();
            }
        }
        if (*abort_flag && lane == 0) {
            // drain: the loads this warp issued land before the CTA exits. The first CTA waits
            // on its stage barriers (bounded); the second cannot wait on the first's barriers and
            // gives its in-flight copies a fixed 200 us
            const uint64_t t0 = globaltimer();
            if (rank == 0) {
                for (int i = max(0, issued - kPStages); i < issued; ++i)
                    while (!mbar_try_wait(BAR(PG_FULL + i % kPStages), (uint32_t)(i / kPStages) & 1u) &&
                           globaltimer() - t0 < kWaitLimitNs) {
                    }
            } else {
                while (globaltimer() - t0 < 200000ull) {
                }
            }
        }
    } else if (warp == kGWarpMMA) {
        // ---------------------------------------------------------------------- MMA issuer
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = instr_desc(256, 0, 256);
            const uint64_t da = smem_desc_sw128(sbase + OFF_PSTAGE, 16, 1024);
            const uint64_t db = smem_desc_sw128(sbase + OFF_PSTAGE + kPABytes, 16, 1024);
            constexpr uint64_t kStageDesc = kPStageBytes >> 4;
            int it = 0, nt = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < n_tiles; tile += n_pairs, ++nt) {
                const int b = nt & 1;
                if (nt >= 2) {  // both CTAs' epilogues have read this accumulator's previous tile
                    if (!wait_bounded(BAR(PG_AEMPTY + b), (uint32_t)((nt >> 1) - 1) & 1u, abort_flag, a.status)) break;
                    tc_fence_after();
                }
                const uint32_t d_t = tmem + (uint32_t)b * kAccCols;
                for (int ks = 0; ks < k_steps; ++ks, ++it) {
                    const int s = it % kPStages;
                    if (!wait_bounded(BAR(PG_FULL + s), (uint32_t)(it / kPStages) & 1u, abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t sa = da + (uint64_t)s * kStageDesc, sb = db + (uint64_t)s * kStageDesc;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        tc_mma_pair(d_t, sa + (uint64_t)(kk * 2), sb + (uint64_t)(kk * 2), idesc, (ks | kk) ? 1u : 0u);
                    tc_commit_pair_both(BAR(PG_EMPTY + s));
                }
                if (!ok) break;
                tc_commit_pair_both(BAR(PG_AFULL + b));
            }
            tc_commit_pair(BAR(PG_DRAIN));
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(BAR(PG_DRAIN), 0) && globaltimer() - t0 < kWaitLimitNs) {
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------------- epilogue
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const bool leader = threadIdx.x == 64;
        const int ft = a.grid_h * a.grid_w;
        const uint32_t aempty0 = mapa_shared(BAR(PG_AEMPTY), 0);  // the first CTA's release barriers
        int nt = 0, slab_n = 0;
        for (int tile = pair; tile < n_tiles; tile += n_pairs, ++nt) {
            const int b = nt & 1;
            int m0, n0;
            if (a.n_major) {
                m0 = (tile % a.n_tiles_m) * 256;
                n0 = (tile / a.n_tiles_m) * 256;
            } else {
                m0 = (tile / a.n_tiles_n) * 256;
                n0 = (tile % a.n_tiles_n) * 256;
            }
            m0 += 128 * (int)rank;  // this CTA's rows of the tile
            const bool got = warp_wait(BAR(PG_AFULL + b), (uint32_t)(nt >> 1) & 1u, abort_flag, a.status);
            uint32_t all_got;
            asm volatile(
                "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                : "=r"(all_got)
                : "r"((uint32_t)got)
                : "memory");
            if (!all_got) break;
            tc_fence_after();
            const int section = n0 / a.hd;
            const int col0 = n0 - section * a.hd;
            const int tok = a.tok0 + min(m0 + row, a.m - 1);
            const int f = tok / ft, rem = tok - f * ft;
            const int t = a.start_frame + f, hh = rem / a.grid_w, ww = rem - hh * a.grid_w;
            for (int sl = 0; sl < kBN / 64; ++sl, ++slab_n) {
                uint32_t v[64];
                tmem_ld32(tmem + lane_base + (uint32_t)b * kAccCols + sl * 64, v);
                tmem_ld32(tmem + lane_base + (uint32_t)b * kAccCols + sl * 64 + 32, v + 32);
                tmem_ld_wait(v);
                reg_touch32(v + 32);
                if (sl == kBN / 64 - 1) {
                    // every column of this CTA's accumulator is in registers: release it
                    tc_fence_before();
                    mbar_arrive_cluster(aempty0 + 8u * (uint32_t)b);
                }
                const int feat0 = col0 + sl * 64;
                if (section < 2) {
                    const int pp0 = (feat0 % a.head_dim) >> 1;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float2 cs = pair_angle(pp0 + i, t, hh, ww, a);
                        const float x0 = __uint_as_float(v[2 * i]), x1 = __uint_as_float(v[2 * i + 1]);
                        v[2 * i] = __float_as_uint(fmaf(x0, cs.x, -x1 * cs.y));
                        v[2 * i + 1] = __float_as_uint(fmaf(x0, cs.y, x1 * cs.x));
                    }
                }
                const int buf = slab_n & 1;
                if (leader) bulk_wait_read<1>();
                asm volatile("bar.sync 1, 128;" ::: "memory");
                uint8_t* stage = smem + OFF_POUT + buf * kOutSlab;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat162 p2 = __floats2bfloat162_rn(__uint_as_float(v[8 * c + 2 * e]),
                                                                  __uint_as_float(v[8 * c + 2 * e + 1]));
                        memcpy(&w4[e], &p2, 4);
                    }
                    *reinterpret_cast<uint4*>(stage + row * 128 + ((c ^ (row & 7)) << 4)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
                fence_proxy_async_smem();
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (leader && m0 < a.m) {
                    const uint32_t src = sbase + OFF_POUT + buf * kOutSlab;
                    if (section == 0)
                        tma_store_2d(&map_q, src, feat0, m0);
                    else
                        tma_store_3d(section == 1 ? &map_k : &map_v, src, feat0 % a.head_dim, m0,
                                     feat0 / a.head_dim);
                }
                if (leader) bulk_commit();
            }
        }
        if (leader) bulk_wait_all();
    }
    // ------------------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the first CTA's MMAs into this CTA's TMEM have completed (its drain)
    if (warp == kGWarpMMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kAccCols)
                     : "memory");
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
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

// bf16 tensor map with the 128-byte swizzle; dims[0] innermost (elements), strides in bytes for
// dims 1.. ; box[0] = 64 elements (128 bytes).
int encode(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
           const cuuint32_t* box) {
    auto enc = encoder();
    if (!enc) return vdit::fail(VDIT_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
                           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? VDIT_OK : vdit::fail(VDIT_ERR_CUDA, "cuTensorMapEncodeTiled failed");
}

// Per-device set-up, once per device with that device current: the kernel's dynamic shared-memory
// opt-in (a function attribute belongs to one device's context), the status word's device
// address and the SM count.
struct QkvDeviceState {
    bool ready = false;
    int* status = nullptr;
    int sms = 148;
};
constexpr int kMaxDevices = 256;
std::mutex g_qkv_dev_mu;
QkvDeviceState g_qkv_dev[kMaxDevices];

int qkv_device_state(int dev, QkvDeviceState* out) {
    if (dev < 0 || dev >= kMaxDevices) return vdit::fail(VDIT_ERR_INVALID_ARG, "device index too large");
    std::lock_guard<std::mutex> lk(g_qkv_dev_mu);
    QkvDeviceState& st = g_qkv_dev[dev];
    if (!st.ready) {
        if (int rc = vdit::cuda_check(cudaFuncSetAttribute(qkv_rope_pair_kernel,
                                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                           (int)kPSmemBytes),
                                      "cudaFuncSetAttribute(qkv_rope_pair)"))
            return rc;
        void* sp = nullptr;
        if (int rc = vdit::cuda_check(cudaGetSymbolAddress(&sp, g_qkv_status), "cudaGetSymbolAddress(status)"))
            return rc;
        st.status = static_cast<int*>(sp);
        if (int rc = vdit::cuda_check(cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev),
                                      "cudaDeviceGetAttribute"))
            return rc;
        st.ready = true;
    }
    *out = st;
    return VDIT_OK;
}

// One launch over `n_tok` consecutive tokens of the chunk (chunk-local first token tok0) whose K
// and V rows go to consecutive cache rows starting at cache_row0.
int launch_part(const vdit_geom* g, const vdit::RopeTables& tabs, const uint8_t* x, const void* w,
                int d_model, int start_frame, int tok0, int n_tok, uint8_t* q, void* k_cache, void* v_cache,
                long long cap_tok, long long cache_row0, const QkvDeviceState& ds, cudaStream_t st) {
    const int hd = g->heads * g->head_dim, d = g->head_dim;
    CUtensorMap mx, mw, mq, mk, mv;
    {
        cuuint64_t dims[2] = {(cuuint64_t)d_model, (cuuint64_t)n_tok};
        cuuint64_t str[1] = {(cuuint64_t)d_model * 2};
        cuuint32_t box[2] = {64, kBM};
        if (int rc = encode(&mx, x + (size_t)tok0 * d_model * 2, 2, dims, str, box)) return rc;
    }
    {
        // each CTA of a pair stages 128 of the 256 W rows of a tile
        cuuint64_t dims[2] = {(cuuint64_t)d_model, (cuuint64_t)3 * hd};
        cuuint64_t str[1] = {(cuuint64_t)d_model * 2};
        cuuint32_t box[2] = {64, 128};
        if (int rc = encode(&mw, w, 2, dims, str, box)) return rc;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)hd, (cuuint64_t)n_tok};
        cuuint64_t str[1] = {(cuuint64_t)hd * 2};
        cuuint32_t box[2] = {64, kBM};
        if (int rc = encode(&mq, q + (size_t)tok0 * hd * 2, 2, dims, str, box)) return rc;
    }
    for (int which = 0; which < 2; ++which) {
        cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n_tok, (cuuint64_t)g->heads};
        cuuint64_t str[2] = {(cuuint64_t)d * 2, (cuuint64_t)cap_tok * d * 2};
        cuuint32_t box[3] = {64, kBM, 1};
        uint8_t* base = static_cast<uint8_t*>(which ? v_cache : k_cache) + (size_t)cache_row0 * d * 2;
        if (int rc = encode(which ? &mv : &mk, base, 3, dims, str, box)) return rc;
    }
    GemmArgs a{};
    a.m = n_tok;
    a.k = d_model;
    a.n_tiles_m = (n_tok + 255) / 256;
    a.n_tiles_n = 3 * hd / kBN;
    a.n_major = (long long)3 * hd > (long long)n_tok ? 1 : 0;  // W larger than X: keep X in L2
    a.hd = hd;
    a.head_dim = d;
    a.tok0 = tok0;
    a.start_frame = start_frame;
    a.grid_h = g->grid_h;
    a.grid_w = g->grid_w;
    a.tt = static_cast<const float2*>(tabs.t);
    a.th = static_cast<const float2*>(tabs.h);
    a.tw = static_cast<const float2*>(tabs.w);
    a.bt2 = g->band_t / 2;
    a.bh2 = g->band_h / 2;
    a.bw2 = g->band_w / 2;
    a.status = ds.status;
    const int tiles = a.n_tiles_m * a.n_tiles_n;
    const int grid = 2 * std::min(tiles, ds.sms / 2);  // clusters of two CTAs, persistent
    qkv_rope_pair_kernel<<<grid, kGThreads, kPSmemBytes, st>>>(mx, mw, mq, mk, mv, a);
    return vdit::cuda_check(cudaGetLastError(), "qkv_rope kernel launch");
}

}  // namespace

namespace vdit {
// Reads and clears this file's device status word (VDIT_OK or VDIT_ERR_TIMEOUT).
int qkv_status_take(int* out) {
    int zero = 0, v = 0;
    if (int rc = cuda_check(cudaMemcpyFromSymbol(&v, g_qkv_status, sizeof(int)), "read status")) return rc;
    if (int rc = cuda_check(cudaMemcpyToSymbol(g_qkv_status, &zero, sizeof(int)), "clear status")) return rc;
    *out = v;
    return VDIT_OK;
}
}  // namespace vdit

extern "C" int vdit_qkv_rope(const vdit_geom* g, const void* x, const void* w, int d_model, int start_frame,
                             int n_frames, void* q, void* k_cache, void* v_cache, int capacity_frames,
                             void* stream) {
    using vdit::fail;
    if (int rc = vdit::check_geom(g)) return rc;
    if (!x || !w || !q || !k_cache || !v_cache) return fail(VDIT_ERR_INVALID_ARG, "NULL pointer");
    auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    if (!al(x) || !al(w) || !al(q) || !al(k_cache) || !al(v_cache))
        return fail(VDIT_ERR_MISALIGNED, "tensor not 16-byte aligned");
    const long long hd = (long long)g->heads * g->head_dim;
    if (hd % kBN != 0) return fail(VDIT_ERR_UNSUPPORTED, "heads * head_dim must be a multiple of 256");
    if (d_model < 8 || d_model % 8 != 0) return fail(VDIT_ERR_INVALID_ARG, "d_model must be a positive multiple of 8");
    if (capacity_frames < 1 || n_frames < 1 || n_frames > capacity_frames)
        return fail(VDIT_ERR_INVALID_ARG, "need 1 <= n_frames <= capacity_frames");
    if (start_frame < 0 || start_frame + n_frames - 1 > VDIT_MAX_FRAME)
        return fail(VDIT_ERR_INVALID_ARG, "frames outside [0, VDIT_MAX_FRAME]");
    const long long ft = (long long)g->grid_h * g->grid_w;
    if (ft * n_frames > (1 << 30)) return fail(VDIT_ERR_UNSUPPORTED, "chunk too large");
    vdit::RopeTables tabs;
    if (int rc = vdit::get_rope_tables(g, &tabs)) return rc;
    int dev = 0;
    if (int rc = vdit::cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
    QkvDeviceState ds;
    if (int rc = qkv_device_state(dev, &ds)) return rc;
    // frames of the chunk go to slots (frame mod capacity): one launch per run of consecutive
    // slots (two when the chunk wraps around the end of the ring)
    const long long cap_tok = ft * capacity_frames;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int f = 0;
    while (f < n_frames) {
        const int slot = (start_frame + f) % capacity_frames;
        const int run = std::min(n_frames - f, capacity_frames - slot);
        if (int rc = launch_part(g, tabs, static_cast<const uint8_t*>(x), w, d_model, start_frame, (int)(f * ft),
                                 (int)(run * ft), static_cast<uint8_t*>(q), k_cache, v_cache, cap_tok,
                                 (long long)slot * ft, ds, st))
            return rc;
        f += run;
    }
    return VDIT_OK;
}
