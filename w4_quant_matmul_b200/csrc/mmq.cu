// mmq.cu -- W4A8 prefill product on the sm_100a int8 tensor cores.
//
// The hipfire HFQ4-G256 MMQ article ("What changed" list) pre-quantises the
// prefill activations to a Q8_1-style int8 block layout and runs a tiled int8
// matrix-matrix product over the 4-bit weights, applying the scales after the
// integer products.  Here:
//
//   P[t][n][b] = sum_{k in block b} q[n][k] * qa[t][k]          (exact int32)
//   y[t][n]    = sum_g ( d[n][g] * sum_{b in g} dx[t][b] * P[t][n][b]
//                        + m[n][g] * sum_{b in g} dx[t][b] * S[t][b] )
//
// Persistent CTAs (one per SM) loop over work units = (128-token x 128-row
// output tile, K slice); the pipeline, barriers and TMEM allocation live for
// the whole launch.  K advances in stages of 128 (four 32-element activation
// blocks); two stages make one 256-group.
//   warp 0      TMA producer: the qa tile (128 x 128 B, 128B-swizzled) and the
//               packed code tile (128 rows x 64 B) into a 3-stage ring, and,
//               ahead of each 256-group, that group's dx and S for the tile's
//               128 tokens (8 x 128 boxes of fp32 / int32) into a 2-slot ring.
//   warp 1      allocates 512 TMEM columns = four 128-column block buffers;
//               one lane issues, per 32-block, a tcgen05.mma.kind::i8 (M=128,
//               N=128, K=32; A = qa as s8, B = the codes as u8) into the
//               buffer of the block's position in the stage, as soon as the
//               epilogue has read that buffer's previous block, and one
//               tcgen05.commit per buffer pair.
//   warps 2-3   unpack each code tile, nibble -> byte, into the 128B-swizzled
//               K-major layout the MMA's shared-memory descriptor expects
//               (tcgen05 has no 4-bit integer kind), and at each group's first
//               stage write the tile's d and m (fp32) into a 4-slot ring.
//   warps 4-11  epilogue: each thread owns one token row (its TMEM lane) and 64
//               weight rows.  It reads each block's words in two 32-column
//               halves, each half's TMEM load issued before the previous
//               half's FMAs (two register sets), releases every buffer as soon
//               as its words are in registers, and frees a stage's
//               shared-memory operands once the stage's last commit has
//               landed.  The partial output row (64 fp32 per thread) lives in
//               shared memory, read and written once per group, which leaves
//               the registers for the second load in flight.  Shared memory
//               (~213 KB) does not depend on K.
//
// Measured on B200 (single-SM microbenchmarks): a 128x128x32 kind::i8 MMA
// occupies the tensor pipe 65 cycles (8000 MAC/clk, the full int8 rate), a
// commit adds ~100 cycles when it follows short MMAs, and TMEM -> registers
// moves ~390 B/clk/SM while the words are consumed by FMAs.  The epilogue
// (one FMA and 4 TMEM bytes per 32 multiply-adds) therefore bounds the kernel,
// not the tensor pipe: commits are per pair of blocks and everything else is
// arranged so that the epilogue warps never wait.
//
// Epilogue arithmetic.  Converting 16384 int32 products per block to float at
// the quarter-rate conversion throughput would cost four times the MMA, so
// no conversion is done.  At the start of each 256-group the tensor core
// seeds every buffer with the integer 2^17 (a kind::i8 MMA over constant u8
// tiles, 32 * 64 * 64, in overwrite mode); buffer r then accumulates block r
// of the group and, in the second stage, block r + 4 on top of it.  With
// |P| <= 32*15*127 = 60960 per block, the words read back,
//   V_r = 2^17 + P_r   and   V_{r+4} = 2^17 + P_r + P_{r+4},
// lie in [9152, 252992] -- as fp32 bits, exact denormals V * 2^-149.  Abel
// summation turns the per-block scaling into one full-rate FMA per element
// per block with per-(token, block) coefficients:
//   sum_b dx_b P_b = sum_{r<4} [ (dx_r - dx_{r+4}) V_r + dx_{r+4} V_{r+4} ]
//                    - 2^17 sum_{r<4} dx_r.
// The coefficients carry a factor 2^e, one e per token for the whole unit,
// chosen from the token's largest block scale so that the products stay
// normal (dx_max 2^e in [2^40, 2^41)); a later group whose scales are 2^24
// times larger lowers e and rescales the partial output.  The bias term
// -2^17 sum dx_r enters as the addend of the group's first FMA, and the
// output row is kept in units of 2^(e-149), so the group end costs two FMAs
// per element, ys += d * acc + m * (sum_b dx_b S_b) (ys in shared memory), and
// the unit end one
// multiply by 2^(149-e).  The exact integer block sums never leave TMEM as
// anything but exact values; the fp32 work is the coefficient differences and
// the accumulation.  Requires |dx| < 2^100 (activations far beyond any
// fp16/bf16 model range would overflow the scaled products).
//
// Registers are rebalanced with setmaxnreg: 64 per thread for warps 0-3, 208
// for the epilogue (128*64 + 256*208 <= 384*168, the launch allotment).
// Work units: the output tiles that fill whole waves of CTAs are one unit
// each; the tiles of a last, partial wave (or all tiles, when they fill less
// than a wave) are split along K into slices that write fp32 partial tiles to
// the caller's workspace; the CTA that finishes a tile last sums the partials
// in slice order (bitwise deterministic) and stores y.
// Programmatic dependent launch: the code tiles of a CTA's first stages and
// the d, m planes are read before the wait for the preceding kernel in the
// stream; the activation tiles, scales and sums after it.
// Every mbarrier wait is bounded; a wait that runs out raises the CTA's abort
// flag and the device error word, all roles drain what they issued, TMEM is
// freed and the CTA returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "common.cuh"

namespace {

constexpr int BM = 128;        // tokens per tile (MMA M, TMEM lanes)
constexpr int BN = 128;        // weight rows per tile (MMA N)
constexpr int BK = 128;        // K elements per pipeline stage
constexpr int KB = 32;         // activation block = MMA K for kind::i8
constexpr int STAGES = 3;
constexpr int NTB = 4;         // TMEM block buffers (BN columns each)
constexpr int NPAIR = NTB / 2; // buffer pairs: the unit of MMA -> epilogue hand-off
constexpr int kRing = 4;       // slots of the per-group d/m ring
constexpr int kScRing = 2;     // slots of the per-group dx/S ring
constexpr int BIAS_BYTES = 128 * KB;  // one constant operand tile of the bias MMA
constexpr int kThreads = 384;              // 4 producer-side warps + 8 epilogue warps
constexpr int kEpiWarps = 8;
constexpr int kEpiCols = BN / (kEpiWarps / 4); // 64 weight rows per epilogue thread
constexpr int A_BYTES = BM * BK;
constexpr int B_BYTES = BN * BK;
constexpr int BP_BYTES = BN * BK / 2;
constexpr int TMEM_COLS = NTB * BN;   // 512
constexpr int kMaxGroups = 512;       // K <= 131072 (shared memory does not depend on K)

static_assert(TMEM_COLS == 512, "TMEM allocation must be a power of two <= 512");

struct Smem {
    static constexpr int a = 0;
    static constexpr int b = a + STAGES * A_BYTES;
    static constexpr int bp = b + STAGES * B_BYTES;
    static constexpr int bias = bp + STAGES * BP_BYTES;  // bias MMA operands (A, B)
    // ring of per-group activation scales and block sums: per slot dx fp32
    // [128 tokens][8] then S int32 [128][8]
    static constexpr int kScSlotBytes = 2 * BM * 8 * 4;
    static constexpr int sc = bias + 2 * BIAS_BYTES;
    static constexpr int dm = sc + kScRing * kScSlotBytes;  // fp32 [kRing][d, m][BN]
    static constexpr int ys = dm + kRing * 2 * BN * 4;      // fp32 [16 col quads][256 threads] float4
    static constexpr int bars = ys + 256 * 64 * 4;          // uint64 barriers
    static constexpr int nbars = 3 * STAGES + NPAIR + NTB + 1 + 2 * kScRing + 2 * kRing;
    static constexpr int misc = bars + nbars * 8;         // tmem base, abort flag, last flag
    static constexpr size_t total = (size_t)misc + 16 + 1024;
};

static_assert(Smem::sc % 128 == 0 && Smem::dm % 16 == 0, "ring slots must be aligned");

struct Params {
    const __half* d;
    const __half* m;
    const float* dx;
    const int32_t* S;
    void* y;
    int M, N, K;
    int out_f32;
    int* err;
    int full_tiles;        // tiles [0, full_tiles) are one unit each (the whole K)
    int tail_splits;       // each later tile is split into this many K slices
    int tiles_n;           // output tiles along N
    int units;             // tiles * splits work units (CTAs loop over them)
    int* counters;         // [tiles] arrival counters (split > 1), zeroed before launch
    float* partials;       // [split tiles][tail_splits][BM][BN] fp32 partial tiles
    int32_t* dump;         // test instantiation only: [M][N][K/32] words read back
};


// ---------------------------------------------------------------------------
// tcgen05 wrappers
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    // K-major, 128-byte swizzle: 8-row core groups 1024 bytes apart.
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// K-major, no swizzle, for the 128 x 32-byte constant tiles of the bias MMA:
// 8-row x 16-byte core matrices, K-neighbours 128 B apart, 8-row groups 256 B
// apart (every byte of these tiles is equal, so only the extent matters).
__device__ __forceinline__ uint64_t smem_desc_plain(uint32_t addr) {
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(128 >> 4) << 16) |
           ((uint64_t)(256 >> 4) << 32) | ((uint64_t)1 << 46);
}

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            w4::smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
        "[%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}


// ---------------------------------------------------------------------------
// kernel
// ---------------------------------------------------------------------------

// Wait for tcgen05.ld results: the registers are named as operands, so that
// the compiler cannot move their uses above the wait.
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;"
        : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
          "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
          "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]),
          "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
          "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]),
          "+r"(r[31])
        :
        : "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Packed fp32x2 helpers for fma.rn.f32x2 (sm_100): two fp32 lanes in a .b64.
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ uint64_t pack_u32x2(uint32_t lo, uint32_t hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}
__device__ __forceinline__ void unpack_f32x2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// d = a * b + d, lane-wise, round to nearest (denormal operands kept)
__device__ __forceinline__ void fma_f32x2(uint64_t& d, uint64_t a, uint64_t b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}

__device__ __forceinline__ float pow2f(int e) {  // 2^e for -126 <= e <= 127
    return __uint_as_float((uint32_t)(e + 127) << 23);
}

// kDump (the test instantiation behind w4a8_mmq_blockdots) also stores every
// word read from TMEM, minus the 2^17 bias, to p.dump.
template <bool kDump>
__global__ void __launch_bounds__(kThreads, 1)
    w4a8_mmq_kernel(const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_dx,
                    const __grid_constant__ CUtensorMap tm_s, const Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment of the operand tiles (128B swizzle atoms).
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sa = smem + Smem::a;
    uint8_t* sb = smem + Smem::b;
    uint8_t* sbp = smem + Smem::bp;
    uint8_t* sc = smem + Smem::sc;
    float* dm_s = reinterpret_cast<float*>(smem + Smem::dm);  // [kRing][d, m][BN]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::bars);
    uint64_t* full = bars;                   // TMA landed (A + packed B)       [STAGES]
    uint64_t* unpacked = full + STAGES;      // B unpacked into the MMA layout  [STAGES]
    uint64_t* sfree = unpacked + STAGES;     // the stage's MMAs are complete   [STAGES]
    uint64_t* tfull = sfree + STAGES;        // TMEM buffer pair written        [NPAIR]
    uint64_t* tempty = tfull + NPAIR;        // TMEM buffer read out            [NTB]
    uint64_t* drain = tempty + NTB;          // final MMA completion
    uint64_t* scfull = drain + 1;            // a group's dx/S landed           [kRing]
    uint64_t* scempty = scfull + kScRing;    // the epilogue has read the slot  [kScRing]
    uint64_t* dmfull = scempty + kScRing;    // a group's d, m written          [kRing]
    uint64_t* dmfree = dmfull + kRing;       // every epilogue warp has read it [kRing]
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + Smem::misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Smem::misc + 4);
    volatile int* last_flag = abort_flag + 1;
    const int G = p.K / 256;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Work unit u -> (tile_m, tile_n, K slice [gb, ge) in groups).  Units
    // [0, full_tiles) are whole tiles; every later tile is split into
    // tail_splits K slices (the last, partial wave of tiles spread over all
    // CTAs).  Units handed to consecutive CTAs share tile_m, i.e. the same
    // activation rows.  split_of gives a unit's (slices of its tile, slice
    // index, index among the split tiles).
    auto split_of = [&](int u, int& ns, int& si, int& pt) {
        if (u < p.full_tiles) {
            ns = 1;
            si = 0;
            pt = 0;
        } else {
            const int v = u - p.full_tiles;
            ns = p.tail_splits;
            si = v % p.tail_splits;
            pt = v / p.tail_splits;
        }
    };
    auto unit_of = [&](int u, int& tm, int& tn, int& gb, int& ge) {
        int ns, si, pt;
        split_of(u, ns, si, pt);
        const int tile = u < p.full_tiles ? u : p.full_tiles + pt;
        tn = tile % p.tiles_n;
        tm = tile / p.tiles_n;
        gb = (int)(((long long)G * si) / ns);
        ge = (int)(((long long)G * (si + 1)) / ns);
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            w4::mbar_init(&full[i], 1);
            w4::mbar_init(&unpacked[i], 2);
            w4::mbar_init(&sfree[i], 1);
        }
        for (int i = 0; i < NPAIR; ++i) w4::mbar_init(&tfull[i], 1);
        for (int i = 0; i < NTB; ++i) w4::mbar_init(&tempty[i], kEpiWarps);
        w4::mbar_init(drain, 1);
        for (int i = 0; i < kScRing; ++i) {
            w4::mbar_init(&scfull[i], 1);
            w4::mbar_init(&scempty[i], kEpiWarps);
        }
        for (int i = 0; i < kRing; ++i) {
            w4::mbar_init(&dmfull[i], 2);
            w4::mbar_init(&dmfree[i], kEpiWarps);
        }
        *abort_flag = 0;
        w4::fence_mbar_init();
    }
    // constant operands of the bias MMA: A = B = 64 (u8), so that over K = 32
    // every accumulator starts at 32 * 64 * 64 = 2^17
    {
        uint32_t* ba = reinterpret_cast<uint32_t*>(smem + Smem::bias);
        for (int i = threadIdx.x; i < 2 * BIAS_BYTES / 4; i += kThreads) ba[i] = 0x40404040u;
        w4::fence_proxy_async_smem();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         w4::smem_u32((const void*)tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 64;");
        if (warp == 0) {
            // ---------------- TMA producer ----------------
            if (w4::elect_one()) {
                w4::prefetch_tmap(&tm_a);
                w4::prefetch_tmap(&tm_b);
                w4::prefetch_tmap(&tm_dx);
                w4::prefetch_tmap(&tm_s);
                int it = 0;  // stages issued
                int gi = 0;  // groups whose scales were issued
                bool ok = true;
                // Under programmatic dependent launch the code tiles of the
                // first stages (weights: they do not depend on the preceding
                // kernel) are requested before the dependency wait; the
                // activation tiles and scales, after it.
                int npre = 0;
                if (blockIdx.x < p.units) {
                    int tmi, tni, gb, ge;
                    unit_of(blockIdx.x, tmi, tni, gb, ge);
                    npre = (ge - gb) * 2 < STAGES ? (ge - gb) * 2 : STAGES;
                    for (int i = 0; i < npre; ++i) {
                        w4::mbar_arrive_expect_tx(&full[i], A_BYTES + BP_BYTES);
                        w4::tma_load_2d(sbp + i * BP_BYTES, &tm_b, &full[i],
                                        (gb * 2 + i) * (BK / 2), tni * BN);
                    }
                }
                pdl_wait();
                for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
                    int tmi, tni, gb, ge;
                    unit_of(u, tmi, tni, gb, ge);
                    // tile origins inside the activation and code tensors (the
                    // tensor maps fill what lies past their ends with zeros)
                    (void)W4_CHECK(tmi * BM < p.M && tni * BN < p.N && 0 <= gb && gb < ge &&
                                       ge <= G,
                                   p.err);
                    for (int kg = gb * 2; kg < ge * 2; ++kg, ++it) {
                        if ((kg & 1) == 0) {
                            // the group's dx and S for the tile's 128 tokens (rows
                            // past M are zero-filled), into slot gi % kScRing
                            const int slot = gi % kScRing;
                            if (!w4::mbar_wait(&scempty[slot], ((uint32_t)(gi / kScRing) & 1u) ^ 1u,
                                               abort_flag, p.err)) {
                                ok = false;
                                break;
                            }
                            uint8_t* dst = sc + slot * Smem::kScSlotBytes;
                            w4::mbar_arrive_expect_tx(&scfull[slot], Smem::kScSlotBytes);
                            w4::tma_load_2d(dst, &tm_dx, &scfull[slot], (kg >> 1) * 8, tmi * BM);
                            w4::tma_load_2d(dst + Smem::kScSlotBytes / 2, &tm_s, &scfull[slot],
                                            (kg >> 1) * 8, tmi * BM);
                            ++gi;
                        }
                        const int s = it % STAGES;
                        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                        if (it >= npre) {
                            if (!w4::mbar_wait(&sfree[s], ph ^ 1u, abort_flag, p.err)) {
                                ok = false;
                                break;
                            }
                            w4::mbar_arrive_expect_tx(&full[s], A_BYTES + BP_BYTES);
                            w4::tma_load_2d(sbp + s * BP_BYTES, &tm_b, &full[s], kg * (BK / 2),
                                            tni * BN);
                        }
                        w4::tma_load_2d(sa + s * A_BYTES, &tm_a, &full[s], kg * BK, tmi * BM);
                    }
                }
                // drain: every issued load must land before the CTA exits
                for (int k = it - STAGES < 0 ? 0 : it - STAGES; k < it; ++k)
                    w4::mbar_wait(&full[k % STAGES], (uint32_t)(k / STAGES) & 1u, nullptr, p.err);
                for (int k = gi - kScRing < 0 ? 0 : gi - kScRing; k < gi; ++k)
                    w4::mbar_wait(&scfull[k % kScRing], (uint32_t)(k / kScRing) & 1u, nullptr, p.err);
            }
        } else if (warp == 1) {
            // ---------------- MMA issuer ----------------
            if (w4::elect_one()) {
                constexpr uint32_t idesc = (2u << 4)             // D: s32
                                           | (1u << 7)           // A: s8
                                           | (0u << 10)          // B: u8
                                           | ((uint32_t)(BN >> 3) << 17)
                                           | ((uint32_t)(BM >> 4) << 24);
                constexpr uint32_t idesc_bias = (2u << 4)        // D: s32, A: u8, B: u8
                                                | ((uint32_t)(BN >> 3) << 17)
                                                | ((uint32_t)(BM >> 4) << 24);
                const uint64_t bias_a = smem_desc_plain(w4::smem_u32(smem + Smem::bias));
                const uint64_t bias_b =
                    smem_desc_plain(w4::smem_u32(smem + Smem::bias + BIAS_BYTES));
                int it = 0;
                bool ok = true;
                for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
                    int tmi, tni, gb, ge;
                    unit_of(u, tmi, tni, gb, ge);
                    for (int kg = gb * 2; kg < ge * 2 && ok; ++kg, ++it) {
                        const int s = it % STAGES;
                        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                        if (!w4::mbar_wait(&full[s], ph, abort_flag, p.err) ||
                            !w4::mbar_wait(&unpacked[s], ph, abort_flag, p.err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a_addr = w4::smem_u32(sa + s * A_BYTES);
                        const uint32_t b_addr = w4::smem_u32(sb + s * B_BYTES);
                        // First half of a 256-group (stage kg even): each buffer is
                        // seeded with the bias before its block; second half: the
                        // block accumulates onto the first half's block in that buffer.
                        const bool seed = (kg & 1) == 0;
#pragma unroll
                        for (int j = 0; j < NPAIR; ++j) {
#pragma unroll
                            for (int qq = 0; qq < 2; ++qq) {
                                const int q = 2 * j + qq;  // block in the stage = buffer
                                // the epilogue has read this buffer's previous block
                                if (!w4::mbar_wait(&tempty[q], ((uint32_t)it & 1u) ^ 1u,
                                                   abort_flag, p.err)) {
                                    ok = false;
                                    break;
                                }
                                tc_fence_after();
                                const uint32_t dt = tmem_base + (uint32_t)(q * BN);
                                if (seed) mma_i8(dt, bias_a, bias_b, idesc_bias, 0u);  // D = 2^17
                                mma_i8(dt, smem_desc_sw128(a_addr + q * KB),
                                       smem_desc_sw128(b_addr + q * KB), idesc, 1u);  // D += P
                            }
                            if (!ok) break;
                            mma_commit(&tfull[j]);
                        }
                    }
                }
                mma_commit(drain);
                w4::mbar_wait(drain, 0u, nullptr, p.err);
            }
        } else {
            // ---------------- unpackers (warps 2, 3) ----------------
            // Per stage: the packed code tile, nibble -> byte, into the 128B-
            // swizzled K-major layout of the MMA's B operand.  Per group: the
            // tile's d and m (fp16 -> fp32) into slot g % kRing of the d/m ring.
            const int ut = threadIdx.x - 64;  // 0..63
            int it = 0;
            int gq = 0;  // groups whose d, m were written
            bool ok = true;
            for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
                int tmi, tni, gb, ge;
                unit_of(u, tmi, tni, gb, ge);
                for (int kg = gb * 2; kg < ge * 2; ++kg, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    const bool group_start = (kg & 1) == 0;
                    float dmv[4];
                    if (group_start) {
                        // issue the group's d, m loads before the unpack: thread ut
                        // owns entries ut + 64 i of [d, m][BN]
                        const int g = kg >> 1;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int v = ut + 64 * i;
                            const int n = tni * BN + (v & (BN - 1));
                            const __half* src = (v >> 7) ? p.m : p.d;
                            dmv[i] = n < p.N ? __half2float(src[(size_t)n * G + g]) : 0.0f;
                        }
                    }
                    if (!w4::mbar_wait(&full[s], ph, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    const uint8_t* src = sbp + s * BP_BYTES;
                    uint8_t* dst = sb + s * B_BYTES;
                    // Each thread converts 16 chunks of 16 codes in four batches
                    // of 4: all of a batch's loads are issued before its first
                    // store (the compiler cannot tell that the packed source
                    // and the unpacked destination never overlap, so a
                    // load-convert-store loop serialised on every store: ~2400
                    // cycles per stage, the whole pipeline's bottleneck).
#pragma unroll 1
                    for (int batch = 0; batch < 4; ++batch) {
                        uint2 pk[4];
#pragma unroll
                        for (int b = 0; b < 4; ++b) {
                            const int item = (batch * 4 + b) * 64 + ut;
                            const int r = item >> 3, jc = item & 7;  // row, 16-code chunk
                            pk[b] = *reinterpret_cast<const uint2*>(src + r * (BK / 2) + jc * 8);
                        }
#pragma unroll
                        for (int b = 0; b < 4; ++b) {
                            const int item = (batch * 4 + b) * 64 + ut;
                            const int r = item >> 3, jc = item & 7;
                            const uint32_t lo0 = pk[b].x & 0x0F0F0F0Fu;
                            const uint32_t hi0 = (pk[b].x >> 4) & 0x0F0F0F0Fu;
                            const uint32_t lo1 = pk[b].y & 0x0F0F0F0Fu;
                            const uint32_t hi1 = (pk[b].y >> 4) & 0x0F0F0F0Fu;
                            uint4 o;
                            o.x = __byte_perm(lo0, hi0, 0x5140);
                            o.y = __byte_perm(lo0, hi0, 0x7362);
                            o.z = __byte_perm(lo1, hi1, 0x5140);
                            o.w = __byte_perm(lo1, hi1, 0x7362);
                            *reinterpret_cast<uint4*>(dst + r * BK + ((jc ^ (r & 7)) << 4)) = o;
                        }
                    }
                    w4::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) w4::mbar_arrive(&unpacked[s]);
                    if (group_start) {
                        const int slot = gq % kRing;
                        // the slot's previous group (gq - kRing) has been read
                        if (!w4::mbar_wait(&dmfree[slot], ((uint32_t)(gq / kRing) & 1u) ^ 1u,
                                           abort_flag, p.err)) {
                            ok = false;
                            break;
                        }
                        float* d_dst = dm_s + slot * 2 * BN;
#pragma unroll
                        for (int i = 0; i < 4; ++i) d_dst[ut + 64 * i] = dmv[i];
                        __syncwarp();
                        if (lane == 0) w4::mbar_arrive(&dmfull[slot]);
                        ++gq;
                    }
                }
            }
        }
    } else {
        // ---------------- epilogue (warps 4..11) ----------------
        asm volatile("setmaxnreg.inc.sync.aligned.u32 208;");
        const int quarter = warp & 3;               // TMEM lane quarter of this warp
        const int cs = (warp - 4) >> 2;             // column slice: kEpiCols weight rows
        const int row = quarter * 32 + lane;        // token row within the tile
        const uint32_t tm_row =
            tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(cs * kEpiCols);

        int it = 0;
        int gi = 0;  // groups started (the slot sequence of both per-group rings)
        bool ok = true;
        for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
            int tmi, tni, g_begin, g_end;
            unit_of(u, tmi, tni, g_begin, g_end);
            const int n0 = tni * BN;
            const int t = tmi * BM + row;
            const bool t_live = t < p.M;

            // ys: the output row slice in units of 2^(e - 149), e per token, set
            // from the token's activation scales (see the file header)
            float acc[kEpiCols];
            // ys lives in shared memory (float4 [column quad][epilogue thread]);
            // the first group end writes it
            float4* ys_s = reinterpret_cast<float4*>(smem + Smem::ys) + (threadIdx.x - 128);
            bool ys_live = false;
            int e = 127;
            float nb = 0.0f, tp = 0.0f;
            float cf[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) cf[i] = 0.0f;
            const int ksteps = (g_end - g_begin) * 2;
            int gcur = 0;
            for (int ks = 0; ks < ksteps && ok; ++ks, ++it) {
                const bool first_half = (ks & 1) == 0;
                if (first_half) {
                    // ---- group set-up from this token's 8 block scales and sums ----
                    const int slot = gi % kScRing;
                    if (!w4::mbar_wait(&scfull[slot], (uint32_t)(gi / kScRing) & 1u, abort_flag,
                                       p.err)) {
                        ok = false;
                        break;
                    }
                    const uint8_t* src = sc + slot * Smem::kScSlotBytes;
                    const float4 a0 = reinterpret_cast<const float4*>(src)[2 * row];
                    const float4 a1 = reinterpret_cast<const float4*>(src)[2 * row + 1];
                    const int4 s0 =
                        reinterpret_cast<const int4*>(src + Smem::kScSlotBytes / 2)[2 * row];
                    const int4 s1 =
                        reinterpret_cast<const int4*>(src + Smem::kScSlotBytes / 2)[2 * row + 1];
                    __syncwarp();
                    if (lane == 0) w4::mbar_arrive(&scempty[slot]);
                    gcur = gi;
                    ++gi;
                    const float dxg[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                    float tsum = 0.0f;  // sum_b dx_b S_b, fixed order
                    tsum = fmaf(a0.x, (float)s0.x, tsum);
                    tsum = fmaf(a0.y, (float)s0.y, tsum);
                    tsum = fmaf(a0.z, (float)s0.z, tsum);
                    tsum = fmaf(a0.w, (float)s0.w, tsum);
                    tsum = fmaf(a1.x, (float)s1.x, tsum);
                    tsum = fmaf(a1.y, (float)s1.y, tsum);
                    tsum = fmaf(a1.z, (float)s1.z, tsum);
                    tsum = fmaf(a1.w, (float)s1.w, tsum);
                    float dmax = 0.0f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) dmax = fmaxf(dmax, dxg[i]);
                    // e_want puts dmax * 2^e_want in [2^40, 2^41); a group whose
                    // scales outgrow the token's current e by 2^24 or more moves
                    // e down and rescales the partial output (e starts at 127)
                    const int ex = (int)((__float_as_uint(dmax) >> 23) & 0xFFu);
                    int e_want = 167 - ex;
                    e_want = e_want < 22 ? 22 : (e_want > 127 ? 127 : e_want);
                    if (e_want + 24 <= e) {
                        const float r = pow2f(e_want - e);
                        if (ys_live) {
#pragma unroll
                            for (int c4 = 0; c4 < kEpiCols / 4; ++c4) {
                                float4 v = ys_s[c4 * 256];
                                v.x *= r; v.y *= r; v.z *= r; v.w *= r;
                                ys_s[c4 * 256] = v;
                            }
                        }
                        e = e_want;
                    }
                    const float pe = pow2f(e);
                    // buffer r holds V_r = 2^17 + P_r after block r and
                    // V_{r+4} = 2^17 + P_r + P_{r+4} after block r + 4, so
                    //   sum_b dx_b P_b = sum_{r<4} (dx_r - dx_{r+4}) V_r + dx_{r+4} V_{r+4}
                    //                    - 2^17 sum_{r<4} dx_r
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        cf[r] = (dxg[r] - dxg[r + 4]) * pe;
                        cf[r + 4] = dxg[r + 4] * pe;
                    }
                    // -2^17 sum_{r<4} dx_r and sum_b dx_b S_b in units of 2^(e-149)
                    nb = -(((dxg[0] + dxg[1]) + (dxg[2] + dxg[3])) * pe) * 0x1p-66f * 0x1p-66f;
                    tp = (tsum * pe) * 0x1p-75f * 0x1p-74f;
                }
                // ---- the stage's 4 blocks as 8 chunks of 32 columns; each chunk's
                // TMEM load is issued before the previous chunk's FMAs (two
                // register sets), so the load latency overlaps the FMAs ----
                if (!w4::mbar_wait(&tfull[0], (uint32_t)it & 1u, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t rva[32], rvb[32];
                tmem_ld32(tm_row, rva);
                const uint64_t nb2 = pack_f32x2(nb, nb);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int q = c >> 1, h = c & 1;  // block (= buffer), 32-column half
                    uint32_t(&cur)[32] = h ? rvb : rva;
                    uint32_t(&nxt)[32] = h ? rva : rvb;
                    tmem_wait_ld_regs(cur);
                    if (h == 1) {
                        // both halves of block q have been read: its buffer is free
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) w4::mbar_arrive(&tempty[q]);
                    }
                    if (c + 1 < 8) {
                        if (c + 1 == 4) {
                            if (!w4::mbar_wait(&tfull[1], (uint32_t)it & 1u, abort_flag, p.err)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            // the second pair's commit covers all of the stage's MMAs:
                            // its shared-memory operands can be refilled
                            if (threadIdx.x == 128) w4::mbar_arrive(&sfree[it % STAGES]);
                        }
                        tmem_ld32(tm_row + (uint32_t)(((c + 1) >> 1) * BN + 32 * ((c + 1) & 1)), nxt);
                    }
                    if constexpr (kDump) {
                        const int blk = (g_begin + (ks >> 1)) * 8 + (first_half ? q : q + 4);
                        if (t_live) {
                            for (int i = 0; i < 32; ++i) {
                                const int n = n0 + cs * kEpiCols + 32 * h + i;
                                if (n < p.N && W4_CHECK(blk < p.K / 32, p.err))
                                    p.dump[((size_t)t * p.N + n) * (size_t)(p.K / 32) + blk] =
                                        (int32_t)cur[i] - (1 << 17);
                            }
                        }
                    }
                    const float k = first_half ? cf[q] : cf[q + 4];
                    const uint64_t k2 = pack_f32x2(k, k);
                    const bool init = first_half && q == 0;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        uint64_t a2 = init ? nb2
                                           : pack_f32x2(acc[32 * h + 2 * i], acc[32 * h + 2 * i + 1]);
                        fma_f32x2(a2, k2, pack_u32x2(cur[2 * i], cur[2 * i + 1]));
                        unpack_f32x2(a2, acc[32 * h + 2 * i], acc[32 * h + 2 * i + 1]);
                    }
                }
                if (!ok) break;
                if (!first_half) {
                    // ---- group end: ys += d * acc + m * sum_b dx_b S_b ----
                    const int slot = gcur % kRing;
                    if (!w4::mbar_wait(&dmfull[slot], (uint32_t)(gcur / kRing) & 1u, abort_flag,
                                       p.err)) {
                        ok = false;
                        break;
                    }
                    const float4* dg = reinterpret_cast<const float4*>(dm_s + slot * 2 * BN +
                                                                       cs * kEpiCols);
                    const float4* mg = dg + BN / 4;
#pragma unroll
                    for (int c4 = 0; c4 < kEpiCols / 4; ++c4) {
                        const float4 dv = dg[c4], mv = mg[c4];
                        float4 y4 = ys_live ? ys_s[c4 * 256] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        y4.x = fmaf(dv.x, acc[4 * c4 + 0], fmaf(mv.x, tp, y4.x));
                        y4.y = fmaf(dv.y, acc[4 * c4 + 1], fmaf(mv.y, tp, y4.y));
                        y4.z = fmaf(dv.z, acc[4 * c4 + 2], fmaf(mv.z, tp, y4.z));
                        y4.w = fmaf(dv.w, acc[4 * c4 + 3], fmaf(mv.w, tp, y4.w));
                        ys_s[c4 * 256] = y4;
                    }
                    ys_live = true;
                    __syncwarp();
                    if (lane == 0) w4::mbar_arrive(&dmfree[slot]);
                }
            }
            // ---- unit end: y = ys * 2^(149 - e), streamed from shared memory
            // four columns at a time (no 64-register copy of the row), stored
            // directly or through the split-K workspace ----
            float kpow = pow2f(149 - e);
            const int nb0 = n0 + cs * kEpiCols;
            bool store = ok && t_live;
            int nsplit, split, tile;
            split_of(u, nsplit, split, tile);
            if (nsplit > 1) {
                // every epilogue thread reaches both barriers, aborted or not
                // (tile: the index among the split tiles)
                // partial tile layout: float4 [column quad][token row], so the 32
                // lanes (consecutive rows) of a warp store 512 contiguous bytes
                if (ok) {
                    float4* mine = reinterpret_cast<float4*>(
                                       p.partials + ((size_t)tile * nsplit + split) * BM * BN) +
                                   (size_t)cs * (kEpiCols / 4) * BM + row;
#pragma unroll 4
                    for (int c4 = 0; c4 < kEpiCols / 4; ++c4) {
                        float4 v = ys_live ? ys_s[c4 * 256] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        v.x *= kpow; v.y *= kpow; v.z *= kpow; v.w *= kpow;
                        mine[(size_t)c4 * BM] = v;
                    }
                }
                __threadfence();
                asm volatile("bar.sync 1, 256;" ::: "memory");
                if (threadIdx.x == 128) {
                    int last = 0;
                    if (!*abort_flag) last = atomicAdd(p.counters + tile, 1) == nsplit - 1;
                    *last_flag = last;
                }
                asm volatile("bar.sync 1, 256;" ::: "memory");
                const bool last = *last_flag != 0;
                store = store && last;
                if (last) {
                    __threadfence();
                    // the slices summed in slice order, back into this thread's
                    // partial-row slots (now in the output's own scale)
                    const float4* base =
                        reinterpret_cast<const float4*>(p.partials + (size_t)tile * nsplit * BM * BN) +
                        (size_t)cs * (kEpiCols / 4) * BM + row;
                    for (int q = 0; q < nsplit; ++q) {
                        const float4* src = base + (size_t)q * (BM * BN / 4);
#pragma unroll
                        for (int h8 = 0; h8 < kEpiCols / 4; h8 += 8) {
                            float4 v[8];  // eight loads in flight
#pragma unroll
                            for (int i = 0; i < 8; ++i) v[i] = __ldcg(src + (size_t)(h8 + i) * BM);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                float4 sum = q == 0 ? make_float4(0.0f, 0.0f, 0.0f, 0.0f)
                                                    : ys_s[(h8 + i) * 256];
                                sum.x += v[i].x; sum.y += v[i].y; sum.z += v[i].z; sum.w += v[i].w;
                                ys_s[(h8 + i) * 256] = sum;
                            }
                        }
                    }
                    ys_live = true;
                    kpow = 1.0f;
                    if (threadIdx.x == 128) p.counters[tile] = 0;  // ready for the next call
                }
            }
            if (store) {
                auto y4 = [&](int c4) {
                    float4 v = ys_live ? ys_s[c4 * 256] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    v.x *= kpow; v.y *= kpow; v.z *= kpow; v.w *= kpow;
                    return v;
                };
                if (p.out_f32) {
                    float* yr = reinterpret_cast<float*>(p.y) + (size_t)t * p.N;
                    if (nb0 + kEpiCols <= p.N && (p.N & 3) == 0) {
#pragma unroll 4
                        for (int c4 = 0; c4 < kEpiCols / 4; ++c4)
                            *reinterpret_cast<float4*>(yr + nb0 + 4 * c4) = y4(c4);
                    } else {
                        for (int c4 = 0; c4 < kEpiCols / 4; ++c4) {
                            const float4 v = y4(c4);
                            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                if (nb0 + 4 * c4 + i < p.N) yr[nb0 + 4 * c4 + i] = vv[i];
                        }
                    }
                } else {
                    __nv_bfloat16* yr = reinterpret_cast<__nv_bfloat16*>(p.y) + (size_t)t * p.N;
                    if (nb0 + kEpiCols <= p.N && (p.N & 7) == 0) {
#pragma unroll 2
                        for (int c8 = 0; c8 < kEpiCols / 8; ++c8) {
                            const float4 a = y4(2 * c8), b = y4(2 * c8 + 1);
                            __nv_bfloat162 h0 = __floats2bfloat162_rn(a.x, a.y);
                            __nv_bfloat162 h1 = __floats2bfloat162_rn(a.z, a.w);
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(b.x, b.y);
                            __nv_bfloat162 h3 = __floats2bfloat162_rn(b.z, b.w);
                            uint4 v;
                            v.x = *reinterpret_cast<uint32_t*>(&h0);
                            v.y = *reinterpret_cast<uint32_t*>(&h1);
                            v.z = *reinterpret_cast<uint32_t*>(&h2);
                            v.w = *reinterpret_cast<uint32_t*>(&h3);
                            *reinterpret_cast<uint4*>(yr + nb0 + 8 * c8) = v;
                        }
                    } else {
                        for (int c4 = 0; c4 < kEpiCols / 4; ++c4) {
                            const float4 v = y4(c4);
                            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                if (nb0 + 4 * c4 + i < p.N)
                                    yr[nb0 + 4 * c4 + i] = __float2bfloat16_rn(vv[i]);
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// host: tensor maps
// ---------------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// 2-D uint8 tensor map over a dense row-major [rows][cols] byte matrix.
bool make_map_u8(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                 uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D tensor map over a dense row-major [rows][cols] matrix of 4-byte elements
// (fp32 dx or int32 S), no swizzle; rows past the end read as zero.
bool make_map_4b(CUtensorMap* map, const void* base, CUtensorMapDataType type, uint64_t cols,
                 uint64_t rows, uint32_t box_cols, uint32_t box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 4};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Usable dynamic shared memory per CTA on sm_100.
constexpr size_t kSmemMax = 227 * 1024;
static_assert(Smem::total <= kSmemMax, "shared memory layout exceeds one CTA's allotment");

// How the output tiles become work units.  Cost model in units of one
// 256-group of MMA work per CTA: waves of units over the SMs times (groups per
// unit + a fixed cost of a unit's fill, drain and epilogue), each K slice
// keeping >= 2 groups.  Two shapes of plan: every tile split into S K slices
// (S = 1: no split), or the full waves of tiles whole and only the tiles of
// the last, partial wave split, so that the last wave is spread over all SMs.
struct UnitPlan {
    int64_t tiles;
    int full_tiles;   // tiles done as one unit each
    int tail_splits;  // K slices of every later tile
    int64_t units;
    int64_t split_tiles() const { return tail_splits > 1 ? tiles - full_tiles : 0; }
};

UnitPlan plan_units(int64_t M, int64_t N, int64_t K, int sms) {
    const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int G = (int)(K / 256);
    constexpr double kFixed = 1.5;  // per unit, in groups
    UnitPlan best{tiles, (int)tiles, 1, tiles};
    double best_cost = 1e30;
    // every tile split into sp slices
    for (int sp = 1; sp <= 16 && sp <= G; ++sp) {
        if (sp > 1 && G / sp < 4) break;
        const int64_t waves = (tiles * sp + sms - 1) / sms;
        const double cost = (double)waves * ((double)G / sp + kFixed) + (sp > 1 ? 0.25 * sp : 0.0);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = UnitPlan{tiles, sp > 1 ? 0 : (int)tiles, sp, tiles * sp};
        }
    }
    // full waves whole, the last partial wave's tiles split
    const int64_t full = tiles / sms * sms;
    const int64_t rest = tiles - full;
    if (full > 0 && rest > 0) {
        int s = (int)(sms / rest);
        if (s > G / 2) s = G / 2;
        if (s > 16) s = 16;
        if (s >= 2) {
            const double cost = (double)(full / sms) * ((double)G + kFixed) +
                                ((double)G / s + kFixed) + 0.25 * s;
            if (cost < best_cost - 1e-9) {
                best_cost = cost;
                best = UnitPlan{tiles, (int)full, s, full + rest * s};
            }
        }
    }
    return best;
}

constexpr size_t kCounterBytesAlign = 256;

size_t counters_bytes(int64_t tiles) {
    return ((size_t)tiles * 4 + kCounterBytesAlign - 1) / kCounterBytesAlign * kCounterBytesAlign;
}

size_t workspace_for(const UnitPlan& pl) {
    const int64_t st = pl.split_tiles();
    if (st == 0) return 0;
    return counters_bytes(st) + (size_t)st * pl.tail_splits * BM * BN * sizeof(float);
}

}  // namespace

extern "C" {

size_t w4a8_mmq_workspace_size(int64_t M, int64_t N, int64_t K) {
    if (M < 1 || N < 1 || K < 256 || K % 256 != 0) return 0;
    (void)w4::check_device();  // fills the SM count when a device is present
    return workspace_for(plan_units(M, N, K, w4::sm_count()));
}

}  // extern "C"

namespace {

// Host checks shared by w4a8_mmq and w4a8_mmq_static, in one order, so that
// both report the same status for the same bad argument.
int validate_mmq(const uint8_t* codes, const uint16_t* d_f16, const uint16_t* m_f16, int64_t N,
                 int64_t K, const int8_t* qa, const float* dx, const int32_t* bsum, int64_t M,
                 const void* y, int out_dtype) {
    if (M < 1 || N < 1 || K < 256 || K % 256 != 0) return W4_ERR_SHAPE;
    if (K / 256 > kMaxGroups || M > (1 << 24) || N > (1 << 24)) return W4_ERR_SHAPE;
    if (out_dtype != W4_OUT_BF16 && out_dtype != W4_OUT_F32) return W4_ERR_SHAPE;
    if (!codes || !d_f16 || !m_f16 || !qa || !dx || !bsum || !y) return W4_ERR_NULL;
    if (!w4::aligned16(codes) || !w4::aligned16(d_f16) || !w4::aligned16(m_f16) ||
        !w4::aligned16(qa) || !w4::aligned16(dx) || !w4::aligned16(bsum) || !w4::aligned16(y))
        return W4_ERR_ALIGN;
    return w4::check_device();
}

}  // namespace

namespace {

// Launch of the product after validate_mmq: tensor maps, split-K workspace,
// one persistent CTA per SM.  dump != nullptr selects the test instantiation.
int launch_mmq(const uint8_t* codes, const uint16_t* d_f16, const uint16_t* m_f16, int64_t N,
               int64_t K, const int8_t* qa, const float* dx, const int32_t* bsum, int64_t M,
               void* y, int out_dtype, void* workspace, size_t ws_bytes, int32_t* dump,
               void* stream) {
    int* err = w4::device_error_word();
    if (!err) return W4_ERR_CUDA;
    const UnitPlan plan = plan_units(M, N, K, w4::sm_count());
    const size_t need = workspace_for(plan);
    const int64_t split_tiles = plan.split_tiles();
    if (need > 0) {
        if (!workspace || ws_bytes < need) return W4_ERR_WORKSPACE;
        if (!w4::aligned16(workspace)) return W4_ERR_ALIGN;
    }

    CUtensorMap ma, mb;
    if (!make_map_u8(&ma, qa, (uint64_t)K, (uint64_t)M, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B))
        return W4_ERR_CUDA;
    if (!make_map_u8(&mb, codes, (uint64_t)K / 2, (uint64_t)N, BK / 2, BN,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
        return W4_ERR_CUDA;

    const size_t smem = Smem::total;
    // dx and S are [M][K/32]: row stride K/8 bytes (a multiple of 16), box 8 x 128
    CUtensorMap mdx, ms;
    if (!make_map_4b(&mdx, dx, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, (uint64_t)K / 32, (uint64_t)M, 8,
                     BM) ||
        !make_map_4b(&ms, bsum, CU_TENSOR_MAP_DATA_TYPE_INT32, (uint64_t)K / 32, (uint64_t)M, 8,
                     BM))
        return W4_ERR_CUDA;
    static thread_local int attr_dev[2] = {-1, -1};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return w4::cuda_fail(e);
    const int which = dump ? 1 : 0;
    if (attr_dev[which] != dev) {
        e = dump ? cudaFuncSetAttribute(w4a8_mmq_kernel<true>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)Smem::total)
                 : cudaFuncSetAttribute(w4a8_mmq_kernel<false>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)Smem::total);
        if (e != cudaSuccess) return w4::cuda_fail(e);
        attr_dev[which] = dev;
    }
    Params prm;
    prm.d = reinterpret_cast<const __half*>(d_f16);
    prm.m = reinterpret_cast<const __half*>(m_f16);
    prm.dx = dx;
    prm.S = bsum;
    prm.y = y;
    prm.M = (int)M;
    prm.N = (int)N;
    prm.K = (int)K;
    prm.out_f32 = out_dtype == W4_OUT_F32;
    prm.err = err;
    prm.full_tiles = plan.full_tiles;
    prm.tail_splits = plan.tail_splits;
    prm.counters = nullptr;
    prm.partials = nullptr;
    prm.dump = dump;
    if (split_tiles > 0) {
        prm.counters = static_cast<int*>(workspace);
        prm.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                                counters_bytes(split_tiles));
        e = cudaMemsetAsync(workspace, 0, (size_t)split_tiles * 4, (cudaStream_t)stream);
        if (e != cudaSuccess) return w4::cuda_fail(e);
    }
    prm.tiles_n = (int)((N + BN - 1) / BN);
    prm.units = (int)plan.units;
    const int grid = prm.units < w4::sm_count() ? prm.units : w4::sm_count();
    // Programmatic dependent launch (the kernel's prologue and its first code
    // tiles overlap the preceding kernel, e.g. the activation quantiser) when
    // no workspace clear precedes the kernel on the stream.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = (cudaStream_t)stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = split_tiles > 0 ? 0 : 1;
    e = dump ? cudaLaunchKernelEx(&cfg, w4a8_mmq_kernel<true>, ma, mb, mdx, ms, prm)
             : cudaLaunchKernelEx(&cfg, w4a8_mmq_kernel<false>, ma, mb, mdx, ms, prm);
    if (e != cudaSuccess) return w4::cuda_fail(e);
    return w4::launch_status();
}


// The dump holds, per (token, row, group), running sums R_r = P_r and
// R_{r+4} = P_r + P_{r+4} (r < 4) as read from TMEM; this turns the second
// half into block products P_{r+4} = R_{r+4} - R_r.
__global__ void blockdots_from_running_sums(int32_t* __restrict__ P, int64_t rows, int G) {
    const int64_t total = rows * (int64_t)G * 4;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t rg = i >> 2;  // (token, row, group)
        const int r = (int)(i & 3);
        int32_t* grp = P + rg * 8;
        grp[r + 4] -= grp[r];
    }
}

}  // namespace

extern "C" {

int w4a8_mmq(const uint8_t* codes, const uint16_t* d_f16, const uint16_t* m_f16, int64_t N,
             int64_t K, const int8_t* qa, const float* dx, const int32_t* bsum, int64_t M,
             void* y, int out_dtype, void* workspace, size_t ws_bytes, void* stream) {
    int rc = validate_mmq(codes, d_f16, m_f16, N, K, qa, dx, bsum, M, y, out_dtype);
    if (rc != W4_OK) return rc;
    return launch_mmq(codes, d_f16, m_f16, N, K, qa, dx, bsum, M, y, out_dtype, workspace,
                      ws_bytes, nullptr, stream);
}

int w4a8_mmq_blockdots(const uint8_t* codes, const uint16_t* d_f16, const uint16_t* m_f16,
                       int64_t N, int64_t K, const int8_t* qa, const float* dx,
                       const int32_t* bsum, int64_t M, void* y, int out_dtype,
                       int32_t* blockdots, size_t bd_bytes, void* workspace, size_t ws_bytes,
                       void* stream) {
    int rc = validate_mmq(codes, d_f16, m_f16, N, K, qa, dx, bsum, M, y, out_dtype);
    if (rc != W4_OK) return rc;
    if (!blockdots) return W4_ERR_NULL;
    if (!w4::aligned16(blockdots)) return W4_ERR_ALIGN;
    if (bd_bytes < (size_t)M * (size_t)N * (size_t)(K / 32) * 4) return W4_ERR_WORKSPACE;
    rc = launch_mmq(codes, d_f16, m_f16, N, K, qa, dx, bsum, M, y, out_dtype, workspace,
                    ws_bytes, blockdots, stream);
    if (rc != W4_OK) return rc;
    const int64_t total = M * N * (K / 256) * 4;
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)w4::sm_count() * 8) blocks = (int64_t)w4::sm_count() * 8;
    blockdots_from_running_sums<<<(int)blocks, 256, 0, (cudaStream_t)stream>>>(
        blockdots, M * N, (int)(K / 256));
    return w4::launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// w4a8_mmq_static: the same product for callers that cannot allocate device
// memory.  The split-K scratch lives in a library-owned static device array
// instead of a caller workspace.
// ---------------------------------------------------------------------------

namespace {

// Every GPU that loads this library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_mmq_static_scratch[W4A8_MMQ_STATIC_SCRATCH_BYTES];

constexpr int kStaticMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_addr[kStaticMaxDevices];

// Device address of the static scratch on the current device.  The host-side
// name of a __device__ array is only a stand-in, so the address is looked up
// once per device (with that device current) and cached.
int static_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return w4::cuda_fail(e);
    if (dev < 0 || dev >= kStaticMaxDevices) return W4_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (!g_static_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_mmq_static_scratch);
        if (e != cudaSuccess) return w4::cuda_fail(e);
        g_static_addr[dev] = p;
    }
    *out = g_static_addr[dev];
    return W4_OK;
}

}  // namespace

extern "C" int w4a8_mmq_static(const uint8_t* codes, const uint16_t* d_f16,
                               const uint16_t* m_f16, int64_t N, int64_t K, const int8_t* qa,
                               const float* dx, const int32_t* bsum, int64_t M, void* y,
                               int out_dtype, void* stream) {
    int rc = validate_mmq(codes, d_f16, m_f16, N, K, qa, dx, bsum, M, y, out_dtype);
    if (rc != W4_OK) return rc;
    const size_t need = w4a8_mmq_workspace_size(M, N, K);
    if (need > (size_t)W4A8_MMQ_STATIC_SCRATCH_BYTES) return W4_ERR_WORKSPACE;
    void* ws = nullptr;
    if (need > 0) {
        rc = static_scratch(&ws);
        if (rc != W4_OK) return rc;
    }
    return w4a8_mmq(codes, d_f16, m_f16, N, K, qa, dx, bsum, M, y, out_dtype, ws, need, stream);
}
