// gemm_ffma.cu -- fp32 GEMM on the CUDA cores (exact fp32 products, fp32
// FMA accumulation), the fp32 kernel of "TileLang ... 高效 GEMM 内核"
// (mhpq.cn), section 3.2: 128 x 128 output tiles, BK = 32 slices along K,
// 256 computing threads; section 3.3: slices staged in shared memory and
// reused, loads overlapped with math, float4 vector reads.
//
// B200 mapping:
//   warp 8      TMA producer: fills a STAGES-deep ring with the A slice
//               (128 rows x 32 floats = 128 B per row, 128-byte swizzle) and
//               the B slice (32 rows x 128 floats, unswizzled), arming full[s].
//   warps 0-7   compute: thread (tm, tn) owns rows tm + 16 i (i < 8) and
//               columns 4 tn + j, 64 + 4 tn + j (j < 4): an 8 x 8 register
//               tile.  Per 4 k-steps it reads 8 float4 of A (one per row,
//               along k) and per k-step 2 float4 of B; each float4 pair feeds
//               64 fp32 FMAs, issued as 32 paired FMAs (fma.rn.f32x2).  The
//               fragments are double-buffered in registers, so the reads for
//               the next k-step overlap the FMAs of this one.  The swizzle
//               makes the A reads of a warp (4 rows, same k chunk) hit 4
//               distinct bank groups.
//   The accumulators go straight to global memory with float4 stores (a
//   warp writes 4 rows x 128 contiguous bytes), clipped at the matrix edge.
#include "ptx.cuh"
#include "tile_sched.h"
#include "host.cuh"
#include "launch.h"

namespace tg {

namespace {

constexpr int BM = 128, BN = 128, BK = 32, STAGES = 4;
constexpr int A_STAGE = BM * BK * 4;     // 16 KB
constexpr int B_STAGE = BK * BN * 4;     // 16 KB
constexpr int COMPUTE_WARPS = 8;
constexpr int THREADS = 32 * (COMPUTE_WARPS + 1);
constexpr int SMEM_BYTES = STAGES * (A_STAGE + B_STAGE) + 256 + 1024;
// Layout guards: the 128-byte-swizzled A stages start on 1024-byte
// boundaries; the barriers and flags fit their 256 bytes; one CTA fits the
// 227 KB limit; the 8 compute warps' 8 x 8 register tiles cover the block.
static_assert(A_STAGE % 1024 == 0 && B_STAGE % 1024 == 0, "stage alignment");
static_assert((2 * STAGES + 2) * 8 + 2 * 4 <= 256, "barrier area");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
static_assert(COMPUTE_WARPS * 32 * 64 == BM * BN, "8 x 8 outputs per compute thread");

struct FfmaParams {
    int M, N, K, ldc;
    int splits;               // k ranges per output tile (blockIdx.z); 1 = no split
    float* ws;                // splits > 1: [tile][split][BM][BN] fp32 partials
    int* tickets;             // splits > 1: [tile], zero between calls
    int relu;
    int inject;               // debug: 1 = CTA (0, 0, 0)'s producer skips arming the first slot
    unsigned long long timeout_ns;
    int* status;
    float* C;
};

__device__ __forceinline__ float4 lds128(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

// The thread's 8 rows of A at 4-step group g of a slice: one float4 per row
// (rows tm + 16 i; 128-byte rows, 16-byte unit g stored at unit g ^ (tm & 7)).
__device__ __forceinline__ void load_a(uint32_t a_base, uint32_t xr, int g, float4 (&a)[8]) {
    const uint32_t off = (static_cast<uint32_t>(g) ^ xr) << 4;
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = lds128(a_base + i * 16 * 128 + off);
}

// The thread's 8 columns of one B row as 4 pairs: columns 4 tn .. 4 tn + 3
// and 64 + 4 tn .. 64 + 4 tn + 3.
__device__ __forceinline__ void load_b(uint32_t brow, uint64_t (&bp)[4]) {
    asm volatile("ld.shared.v2.u64 {%0, %1}, [%2];" : "=l"(bp[0]), "=l"(bp[1]) : "r"(brow));
    asm volatile("ld.shared.v2.u64 {%0, %1}, [%2];" : "=l"(bp[2]), "=l"(bp[3]) : "r"(brow + 256));
}

__global__ void __launch_bounds__(THREADS, 1)
ffma_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                 const __grid_constant__ CUtensorMap tmB,
                 const FfmaParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* smA = smem;
    uint8_t* smB = smA + STAGES * A_STAGE;
    uint64_t* full = reinterpret_cast<uint64_t*>(smB + STAGES * B_STAGE);
    uint64_t* empty = full + STAGES;
    uint64_t* join = empty + STAGES;                   // compute warps meet (split-K)
    uint64_t* flag = join + 1;                         // ticket result published
    volatile int* abort_flag = reinterpret_cast<volatile int*>(flag + 1);
    volatile int* last_flag = abort_flag + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // this CTA's slices: [kb0, kb0 + num_kb) of the tile's k range
    const int kb_all = (p.K + BK - 1) / BK;
    const int kb_per = ffma_kb_per(kb_all, p.splits);
    const int kb0 = static_cast<int>(blockIdx.z) * kb_per;
    const int num_kb = ffma_range_len(kb0, kb_per, kb_all);
    const int m0 = blockIdx.y * BM;
    const int n0 = blockIdx.x * BN;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], COMPUTE_WARPS);
        }
        mbar_init(join, COMPUTE_WARPS);
        mbar_init(flag, 1);
        *abort_flag = 0;
        *last_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    __syncthreads();

    if (warp == COMPUTE_WARPS) {
        // ---------------------------------------------------- TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            uint32_t armed = 0, armed_par = 0;
            bool ok = true;
            for (int kb = 0; kb < num_kb; ++kb) {
                const int s = kb % STAGES;
                const uint32_t ph = (kb / STAGES) & 1;
                if (!bounded_wait(&empty[s], ph ^ 1, abort_flag, p.timeout_ns, p.status)) {
                    ok = false;
                    break;
                }
                if (p.inject == 1 && kb == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
                    continue;                                   // debug: never arm slot 0
                mbar_arrive_expect_tx(&full[s], A_STAGE + B_STAGE);
                armed |= 1u << s;
                armed_par = (armed_par & ~(1u << s)) | (ph << s);
                tma_load_2d(smA + s * A_STAGE, &tmA, &full[s], (kb0 + kb) * BK, m0);
                tma_load_2d(smB + s * B_STAGE, &tmB, &full[s], n0, (kb0 + kb) * BK);
            }
            if (!ok) {
                for (int s = 0; s < STAGES; ++s)
                    if (armed & (1u << s)) {
                        volatile int never = 0;
                        bounded_wait(&full[s], (armed_par >> s) & 1, &never, p.timeout_ns, p.status);
                    }
            }
        }
        return;
    }

    // -------------------------------------------------------- compute warps
    const int tm = (warp >> 1) * 4 + (lane >> 3);     // 0..15
    const int tn = (warp & 1) * 8 + (lane & 7);       // 0..15
    const uint32_t xr = static_cast<uint32_t>(tm & 7); // swizzle phase of all 8 rows
    // Accumulators are register pairs acc2[i][jp] = (C[i][2 jp], C[i][2 jp + 1])
    // updated with the paired fp32 FMA (fma.rn.f32x2): each instruction does
    // two independent fp32 FMAs, rounded exactly as two scalar FFMAs, and
    // halves the issue slots the math needs.
    uint64_t acc2[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc2[i][j] = 0ull;

    const uint32_t a_base0 = smem_u32(smA) + tm * 128;
    const uint32_t b_base0 = smem_u32(smB) + tn * 16;
    // Register fragments are double-buffered: while the paired FMAs of k-step
    // k issue, the A values of the next 4-step group and the B pairs of k + 1
    // are already being read; at a slice's last k-step the first fragments of
    // the next slice are read, so the math never waits on shared memory.
    float4 a[2][8];          // [buffer][row i]: A[row][4 g .. 4 g + 3]
    uint64_t bp[2][4];       // [buffer][pair j]: (B[k][2 j'], B[k][2 j' + 1])
    if (num_kb > 0) {
        if (!bounded_wait(&full[0], 0, abort_flag, p.timeout_ns, p.status)) return;
        load_a(a_base0, xr, 0, a[0]);
        load_b(b_base0, bp[0]);
    }
    for (int kb = 0; kb < num_kb; ++kb) {
        const int s = kb % STAGES;
        const uint32_t a_base = a_base0 + s * A_STAGE;
        const uint32_t b_base = b_base0 + s * B_STAGE;
        bool ok = true;
#pragma unroll
        for (int k = 0; k < BK; ++k) {
            if (k + 1 < BK) {
                if (((k + 1) & 3) == 0) load_a(a_base, xr, (k + 1) >> 2, a[((k + 1) >> 2) & 1]);
                load_b(b_base + (k + 1) * (BN * 4), bp[(k + 1) & 1]);
            } else if (kb + 1 < num_kb) {
                const int s2 = (kb + 1) % STAGES;
                ok = bounded_wait(&full[s2], ((kb + 1) / STAGES) & 1, abort_flag, p.timeout_ns, p.status);
                if (ok) {
                    load_a(a_base0 + s2 * A_STAGE, xr, 0, a[0]);
                    load_b(b_base0 + s2 * B_STAGE, bp[0]);
                }
            }
            const float4 (&ak)[8] = a[(k >> 2) & 1];
            const uint64_t (&bk)[4] = bp[k & 1];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float av = (k & 3) == 0 ? ak[i].x : (k & 3) == 1 ? ak[i].y : (k & 3) == 2 ? ak[i].z : ak[i].w;
                uint64_t aa;
                asm("mov.b64 %0, {%1, %1};" : "=l"(aa) : "f"(av));
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc2[i][j]) : "l"(aa), "l"(bk[j]));
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (!ok) break;
    }
    if (*abort_flag) return;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            asm("mov.b64 {%0, %1}, %2;" : "=f"(acc[i][2 * j]), "=f"(acc[i][2 * j + 1]) : "l"(acc2[i][j]));

    // ---------------------------------------------------------- epilogue
    // C[row][col .. col + 3] = epi(v), clipped at the matrix edge
    auto store4 = [&](int row, int col, float4 q) {
        if (row >= p.M) return;
        float v[4] = {q.x, q.y, q.z, q.w};
        if (p.relu)
#pragma unroll
            for (int j = 0; j < 4; ++j) v[j] = fmaxf(v[j], 0.f);
        float* crow = p.C + static_cast<size_t>(row) * p.ldc;
        if (col + 3 < p.N) {
            *reinterpret_cast<float4*>(crow + col) = make_float4(v[0], v[1], v[2], v[3]);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (col + j < p.N) crow[col + j] = v[j];
        }
    };
    if (p.splits == 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                store4(m0 + tm + 16 * i, n0 + h * 64 + tn * 4,
                       make_float4(acc[i][h * 4], acc[i][h * 4 + 1], acc[i][h * 4 + 2], acc[i][h * 4 + 3]));
        return;
    }
    // Split K: publish this k range's partial tile and take the tile's
    // ticket; the CTA of the last range adds the partials in range order
    // (deterministic) and writes C.  The compute warps meet on mbarriers
    // with bounded waits.
    const int tile = blockIdx.y * gridDim.x + blockIdx.x;
    float* part = p.ws + (static_cast<size_t>(tile) * p.splits + blockIdx.z) * (BM * BN);
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h)
            *reinterpret_cast<float4*>(part + (tm + 16 * i) * BN + h * 64 + tn * 4) =
                make_float4(acc[i][h * 4], acc[i][h * 4 + 1], acc[i][h * 4 + 2], acc[i][h * 4 + 3]);
    __threadfence();
    __syncwarp();
    if (lane == 0) mbar_arrive(join);
    if (!bounded_wait(join, 0, abort_flag, p.timeout_ns, p.status)) return;
    if (threadIdx.x == 0) {
        const int old = atomicAdd(&p.tickets[tile], 1);
        const int last = old == p.splits - 1;
        if (last) atomicExch(&p.tickets[tile], 0);
        *last_flag = last;
        mbar_arrive(flag);
    }
    if (!bounded_wait(flag, 0, abort_flag, p.timeout_ns, p.status)) return;
    if (!*last_flag) return;
    __threadfence();
    const float* base = p.ws + static_cast<size_t>(tile) * p.splits * (BM * BN);
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int off = (tm + 16 * i) * BN + h * 64 + tn * 4;
            float4 v = __ldcg(reinterpret_cast<const float4*>(base + off));
            for (int z = 1; z < p.splits; ++z) {
                const float4 x = __ldcg(reinterpret_cast<const float4*>(base + static_cast<size_t>(z) * (BM * BN) + off));
                v.x += x.x; v.y += x.y; v.z += x.z; v.w += x.w;
            }
            store4(m0 + tm + 16 * i, n0 + h * 64 + tn * 4, v);
        }
}

}  // namespace

int launch_ffma_f32(const GemmArgs& a) {
    // size limits of this kernel, refused before any CUDA call: a 32-bit
    // output pitch, and at most 65535 tile rows (grid.y)
    if (a.ldc > 0x7fffffff || (a.M + BM - 1) / BM > 65535) return kUnsupported;
    int dev = 0;
    if (!current_device(&dev)) return kNoDevice;
    CUtensorMap tA, tB;
    if (!tensor_map_2d(&tA, a.A, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.K, a.M, a.lda * 4,
                       BK, BM, SWZ_128))
        return kCudaError;
    if (!tensor_map_2d(&tB, a.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.N, a.K, a.ldb * 4,
                       BN, BK, SWZ_NONE))
        return kCudaError;
    if (set_smem_attr(reinterpret_cast<const void*>(ffma_gemm_kernel), SMEM_BYTES, 8) != cudaSuccess)
        return kCudaError;
    const DeviceInfo* di = current_device(&dev);
    const long long tiles_n = (a.N + BN - 1) / BN, tiles_m = (a.M + BM - 1) / BM;
    const long long tiles = tiles_n * tiles_m;
    const long long kb_all = (a.K + BK - 1) / BK;
    // Fewer output tiles than SMs: split K so the grid fills the chip (or
    // the tuning rule's split count, trimmed so that no k range is empty).
    long long splits = ffma_splits(tiles, kb_all, di->num_sms);
    if (a.splits > 0) {
        const long long s = a.splits < kb_all ? a.splits : kb_all;
        const long long per = (kb_all + s - 1) / s;
        splits = (kb_all + per - 1) / per;
    }
    int* tickets = nullptr;
    float* ws = nullptr;
    if (splits > 1 &&
        !stream_workspace(dev, a.stream, tiles, tiles * splits * BM * BN * 4, &tickets, &ws))
        return kCudaError;
    FfmaParams p;
    p.splits = static_cast<int>(splits);
    p.ws = ws;
    p.tickets = tickets;
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.K = static_cast<int>(a.K);
    p.ldc = static_cast<int>(a.ldc);
    p.relu = a.relu;
    p.inject = inject_mode();
    p.timeout_ns = wait_limit_ns();
    p.status = device_status_ptr();
    p.C = static_cast<float*>(a.C);
    if (!p.status) return kCudaError;
    dim3 grid(static_cast<unsigned>(tiles_n), static_cast<unsigned>(tiles_m), static_cast<unsigned>(splits));
    ffma_gemm_kernel<<<grid, THREADS, SMEM_BYTES, static_cast<cudaStream_t>(a.stream)>>>(tA, tB, p);
    return cudaGetLastError() == cudaSuccess ? kOk : kCudaError;
}

}  // namespace tg
