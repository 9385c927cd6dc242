// gemm_w4a16.cu -- grouped expert GEMMs with 4-bit weights and bf16
// activations on the sm_100a tensor cores, the weights decoded into tensor
// memory.
//
// The weights are held at 4 bits ("Mixture of Experts: Why Mixtral Only Wakes
// Up Two Specialists", Part 4, "Why total and active both matter": the model
// loaded in 4-bit precision) as E2M1 codes with an E4M3 scale per 16
// reduction rows and an fp32 scale per matrix (moe_quantize_weights_fp4); the
// activations stay bf16.  The product is the SwiGLU expert of the layer
// equation ("Mixtral of Experts" section 2.1), run on the rows routed to each
// expert:
//   GEMM1: H[r] = bf16( silu(st1 Xp[r] . W1[e]) * (st3 Xp[r] . W3[e]) )
//   GEMM2: O[r] = bf16( st2 H[r] . W2[e] )
// with W = E2M1(code) * sb exactly representable in bf16.
//
// Why this layout.  The tensor core reads operand A from tensor memory, so
// the weights are that operand (M = 128 weight columns, one per TMEM lane) and
// the activations are B (N = a block of tokens, from shared memory by TMA).
// Decoded weights then never pass through shared memory: shared memory
// carries only the 4-bit codes (0.56 bytes per weight) and the activation
// tiles, and the decode writes bf16 pairs straight into tensor memory with
// tcgen05.st.
//
// Packed weights (moe_pack_weights_w4a16): per (expert, tile of 128 packed
// columns, 64 reduction rows) one 4,608-byte block: 4,096 bytes of codes as
// [2 halves][128 columns][16 bytes] (half h = rows 32h .. 32h+31 of the
// step, four 32-bit words of 8 rows each) and 512 bytes of block scales as
// [128 columns][4 E4M3 codes].  GEMM1 uses the gate/up pair layout: packed
// column p of tile j is column 64 j + p of w1 for p < 64 and column
// 64 j + p - 64 of w3 otherwise, so one tile yields both projections of 64
// hidden columns.  A 32-bit word holds 8 consecutive rows k0..k7 as four pairs
// (k0,k1) (k2,k3) (k4,k5) (k6,k7); pair i decodes to one bf16x2 word (lower
// row in the low half) by rotating the word right by 0, 4 or 10 bits (pairs
// 0-2; pair 3 takes two rotations, 6 and 14) and masking
// 0x81C081C0: each code's exponent and mantissa bits land in the bf16's lowest
// two exponent bits and highest mantissa bit, its sign in the sign bit, which
// makes the bf16 value exactly E2M1(code) * 2^-126 (the zero exponent of the
// 0 and 0.5 codes gives the bf16 subnormals 0 and 2^-127).  One bf16x2
// multiply by sb * 2^118 (exact: at most 6 significant bits) gives
// E2M1(code) * sb * 2^-8, and the epilogue multiplies the fp32 accumulators
// by st * 2^8.
//
// Design (persistent, one CTA per SM, 15 warps):
//   warp 12     weight producer: one cp.async.bulk of a 4,608-byte block per
//               stage into a deep ring (DRAM latency under full load is about
//               3 us; a shallow ring tied to the TMEM slots held the decode
//               layer to 0.2 ms for 0.53 GB before any decoding was done).
//   warp 13     activation producer: the kBN x 64 activation tile of each
//               stage (TMA, 128-byte swizzle) into a short ring (L2 hits).
//   warps 4-11  decoders, two per TMEM lane quarter (alternate stages): each
//               thread is one packed column; it reads its 32 code bytes and 4
//               scales, decodes 64 weights into 32 bf16x2 words and stores
//               them to the stage's A slot in tensor memory (32 columns).
//   warp 14     allocates TMEM; one thread issues tcgen05.mma (A from TMEM,
//               B from shared memory, M = 128, N = kBN, K = 16) and frees the
//               A slot and the activation stage with tcgen05.commit.
//   warps 0-3   epilogue: tcgen05.ld of the accumulator (thread = packed
//               column, registers = tokens); GEMM1 exchanges the w3 half
//               through shared memory and applies silu(a) * b; bf16 stores.
// TMEM: two kBN-column accumulators, then one 32-column A slot per stage in
// flight.
// Every wait is bounded (common.cuh).
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kW16Cols = 128;              // packed columns per tile (MMA M)
constexpr int kW16K = 64;                  // reduction rows per stage
constexpr int kW16CodeBytes = 4096;        // 128 columns x 64 rows x 4 bits
constexpr int kW16BlockBytes = kW16CodeBytes + 512;
constexpr int kDecGroups = 2;  // decoder groups of 4 warps, taking stages in turn

constexpr int kWeightWarp = 4 + 4 * kDecGroups;   // producer of the weight ring
constexpr int kActWarp = 5 + 4 * kDecGroups;      // producer of the activation ring
constexpr int kMmaWarp = 6 + 4 * kDecGroups;
constexpr uint32_t kPairMask = 0x81C081C0u;
constexpr int kMaxRing = 8;

// A stage is kBlocks 64-row reduction blocks, moved by ONE copy per ring:
// the weight blocks of consecutive reduction steps are adjacent in the pack,
// and the activation tile comes through a 3-D map (64 columns, rows, 64-column
// chunk) whose box holds kBlocks chunks.  Small copies are what limit a TMA
// pipeline (about 250 cycles each here, however small): one copy per 4.6 KB
// held the decode layer to 2.6 TB/s before any decoding was done.
// Three rings, each sized for what feeds it: weight blocks come from DRAM
// (deep ring), activation tiles are re-read from L2 by every weight tile of an
// expert (short ring), and the decoded weights sit in TMEM A slots, which need
// only cover the MMA's lag behind the decoders.  TMEM: two kBN-column
// accumulators, then the A slots (32 columns per block).
template <int kBN>
struct W16Cfg {
    static constexpr int kBlocks = kBN == 32 ? 4 : 2;        // 64-row blocks per stage
    // MMA issuers: a tcgen05.mma costs its issuing thread about 90 cycles at
    // N = 32 whatever the operands, so at decode two warps issue alternate
    // stages, each into its own accumulator, and the epilogue adds the two
    // (measured: 1.45x the issue rate of one thread).  N = 128 MMAs do 4x
    // the work per instruction, and TMEM has room for one issuer's pair of
    // accumulators only.
    static constexpr int kIssuers = kBN == 32 ? 2 : 1;
    static constexpr int kThreads = (4 + 4 * kDecGroups + 2 + kIssuers) * 32;
    static constexpr int kAccCols = 2 * kIssuers * kBN;  // [buffer][issuer] accumulators
    static constexpr int kSlotCols = 32 * kBlocks;
    static constexpr int kASlots = (512 - kAccCols) / kSlotCols;  // 3 (kBN 32) or 4 (kBN 128)
    static constexpr int kActStages = 3;
    static constexpr int kWStages = 8;
    static constexpr int kBBytes = kBN * 128 * kBlocks;      // kBlocks chunks of kBN rows x 64 bf16
    static constexpr int kWStageBytes = kW16BlockBytes * kBlocks;
    static constexpr int kActBytes = kActStages * kBBytes;
    static constexpr int kWBytes = kWStages * kWStageBytes;
    static constexpr int kXbufBytes = kBN * 64 * 4;          // GEMM1: w3 half of the accumulator, fp32
};

struct __align__(8) W16Tail {
    uint64_t wfull[kMaxRing];
    uint64_t wempty[kMaxRing];
    uint64_t xfull[kMaxRing];
    uint64_t xempty[kMaxRing];
    uint64_t afull[kMaxRing];
    uint64_t aempty[kMaxRing];
    uint64_t accum_full[2];
    uint64_t accum_empty[2];
    uint64_t done;
    uint32_t tmem_base;
    int32_t off[257];
    int32_t mblk[257];
};
constexpr int kW16TailBytes = (static_cast<int>(sizeof(W16Tail)) + 127) / 128 * 128;

template <int kBN>
constexpr int w16_smem_bytes() {
    return W16Cfg<kBN>::kActBytes + W16Cfg<kBN>::kWBytes + W16Cfg<kBN>::kXbufBytes + kW16TailBytes + 1024;
}
static_assert(W16Cfg<32>::kWStages <= kMaxRing && W16Cfg<128>::kWStages <= kMaxRing, "ring sizes");
static_assert(W16Cfg<32>::kASlots <= kMaxRing && W16Cfg<32>::kActStages <= kMaxRing, "ring sizes");
static_assert(w16_smem_bytes<32>() <= 232448 && w16_smem_bytes<128>() <= 232448, "shared memory");

struct W16Tile {
    int e, j, row0, rows;
};

__device__ __forceinline__ W16Tile w16_tile(int t, const int32_t* off, const int32_t* mblk, int n, int n_tiles,
                                            int bn) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (mblk[mid] * n_tiles <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    const int local = t - mblk[lo] * n_tiles;
    const int mb = mblk[lo + 1] - mblk[lo];
    W16Tile ti;
    ti.e = lo;
    ti.j = local / mb;
    ti.row0 = off[lo] + (local - ti.j * mb) * bn;
    ti.rows = min(bn, off[lo + 1] - ti.row0);
    return ti;
}

__device__ __forceinline__ uint32_t rotr32(uint32_t x, int s) { return __funnelshift_r(x, x, s); }

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// bf16 of (E4M3 value of `code`) * 2^118 in both halves.  Exact: an E4M3
// value has at most 4 significant bits, so the fp32 product's low 16 bits are
// zero and truncating to bf16 loses nothing.
__device__ __forceinline__ uint32_t scale_pair(uint32_t code) {
    const __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code & 0xFFu), __NV_E4M3);
    const float f = __half2float(__half(hr)) * 0x1p118f;
    const uint32_t b = __float_as_uint(f) >> 16;
    return b | (b << 16);
}

// Decode one packed word (8 rows of one column) into 4 bf16x2 words.
__device__ __forceinline__ void decode_word(uint32_t w, uint32_t sc, uint32_t* out) {
    out[0] = mul_bf16x2(w & kPairMask, sc);
    out[1] = mul_bf16x2(rotr32(w, 4) & kPairMask, sc);
    out[2] = mul_bf16x2(rotr32(w, 10) & kPairMask, sc);
    out[3] = mul_bf16x2((rotr32(w, 6) & 0x81808180u) | (rotr32(w, 14) & 0x00400040u), sc);
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16 (bf16, fp32 accumulate).
__device__ __forceinline__ void tc_mma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                  uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 accumulator columns from taddr, plus (when `second`) the same columns of
// the second issuer's accumulator kBN columns further on, added in fp32.
template <int kIssuers, int kBN>
__device__ __forceinline__ void ld_acc(uint32_t taddr, uint32_t (&r)[32], bool second) {
    tmem_ld_32x32b_x32(taddr, r);
    if (kIssuers > 1 && second) {
        uint32_t r2[32];
        tmem_ld_32x32b_x32(taddr + kBN, r2);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) + __uint_as_float(r2[k]));
    } else {
        tmem_wait_ld();
    }
}

// Named barrier 1 over the four epilogue warps (threads 0-127).
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// The same barrier, returning whether `v` holds on all four epilogue warps, so
// that they leave the tile loop together.
__device__ __forceinline__ bool epi_all(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v))
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float silu_w16(float a) { return a / (1.f + __expf(-a)); }

// kSwiGLU: GEMM1 over the gate/up pair pack (64 hidden columns per tile);
// else GEMM2 (128 output columns per tile).  kBN: tokens per tile (MMA N).
template <bool kSwiGLU, int kBN>
__global__ void __launch_bounds__(W16Cfg<kBN>::kThreads, 1)
    w4a16_gemm_kernel(const __grid_constant__ CUtensorMap tm_act, const W4a16GemmArgs args) {
    using C = W16Cfg<kBN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* act_ring = smem;                         // 1 KB-aligned swizzled tiles
    uint8_t* w_ring = smem + C::kActBytes;            // kBlocks weight blocks of 4,608 bytes per stage
    float* xbuf = reinterpret_cast<float*>(w_ring + C::kWBytes);
    W16Tail* tail = reinterpret_cast<W16Tail*>(w_ring + C::kWBytes + C::kXbufBytes);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n = args.n;
    int* status = args.status;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kWStages; ++s) {
            mbar_init(smem_u32(&tail->wfull[s]), 1);
            mbar_init(smem_u32(&tail->wempty[s]), 4);  // the 4 decoder warps of the stage's group
        }
        for (int s = 0; s < C::kActStages; ++s) {
            mbar_init(smem_u32(&tail->xfull[s]), 1);
            mbar_init(smem_u32(&tail->xempty[s]), 1);  // MMA commit
        }
        for (int s = 0; s < C::kASlots; ++s) {
            mbar_init(smem_u32(&tail->afull[s]), 4);   // the 4 decoder warps
            mbar_init(smem_u32(&tail->aempty[s]), 1);  // MMA commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&tail->accum_full[b]), C::kIssuers);
            mbar_init(smem_u32(&tail->accum_empty[b]), 4);
        }
        mbar_init(smem_u32(&tail->done), C::kIssuers);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == kActWarp && lane == 0) tma_prefetch_desc(&tm_act);
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(&tail->tmem_base), 512);
        tmem_relinquish();
    }
    griddep_wait();
    for (int i = threadIdx.x; i <= n; i += C::kThreads) {
        tail->off[i] = args.offsets[i];
        tail->mblk[i] = args.mblk_base[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tail->tmem_base;
    const int total_tiles = tail->mblk[n] * args.n_tiles;
    const int stride = args.balanced ? balanced_ctas(total_tiles, static_cast<int>(gridDim.x))
                                     : static_cast<int>(gridDim.x);
    const int first = static_cast<int>(blockIdx.x) < stride ? static_cast<int>(blockIdx.x) : total_tiles;
    const int kb_n = args.k_blocks;

    if (warp == kWeightWarp || warp == kActWarp) {
        // ---------------- producers: one ring each ----------------
        if (lane == 0) {
            const bool weights = warp == kWeightWarp;
            const int ring = weights ? C::kWStages : C::kActStages;
            uint64_t* full = weights ? tail->wfull : tail->xfull;
            uint64_t* empty = weights ? tail->wempty : tail->xempty;
            uint32_t i = 0;
            bool ok = true;
            for (int t = first; t < total_tiles && ok; t += stride) {
                const W16Tile ti = w16_tile(t, tail->off, tail->mblk, n, args.n_tiles, kBN);
                const uint8_t* wsrc =
                    args.wpack + (static_cast<int64_t>(ti.e) * args.n_tiles + ti.j) * kb_n * kW16BlockBytes;
                for (int kb = 0; kb < kb_n; kb += C::kBlocks, ++i) {
                    const int slot = static_cast<int>(i % ring);
                    const uint32_t ph = (i / ring) & 1u;
                    if (!mbar_wait(smem_u32(&empty[slot]), ph ^ 1u, status, kStatusTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full[slot]);
                    if (weights) {
                        const uint32_t bytes = static_cast<uint32_t>(min(C::kBlocks, kb_n - kb)) * kW16BlockBytes;
                        mbar_arrive_expect_tx(fb, bytes);
                        bulk_load(smem_u32(w_ring + slot * C::kWStageBytes),
                                  wsrc + static_cast<int64_t>(kb) * kW16BlockBytes, bytes, fb);
                    } else {
                        // the box always lands kBlocks chunks (zeros past K)
                        mbar_arrive_expect_tx(fb, C::kBBytes);
                        tma_load_3d(smem_u32(act_ring + slot * C::kBBytes), &tm_act, fb, 0, ti.row0, kb);
                    }
                }
            }
            // Drain: no copy may still be writing shared memory when the CTA exits.
            // The last min(i, ring) stages were armed; wait for each one's phase.
            const uint32_t armed = i < static_cast<uint32_t>(ring) ? i : static_cast<uint32_t>(ring);
            for (uint32_t k = i - armed; k < i; ++k)
                mbar_wait(smem_u32(&full[k % ring]), (k / ring) & 1u, status, kStatusTimeoutDrain);
        }
    } else if (warp >= kMmaWarp && warp < kMmaWarp + C::kIssuers) {
        if (lane == 0) {
            // issuer j takes the stages s of each tile with s % kIssuers == j
            const int j = warp - kMmaWarp;
            constexpr uint32_t idesc = make_idesc_bf16(kW16Cols, kBN, 0, 0);
            uint32_t i = 0;
            int local = 0;
            bool ok = true;
            for (int t = first; t < total_tiles && ok; t += stride, ++local) {
                const int buf = local & 1;
                const uint32_t bph = static_cast<uint32_t>(local >> 1) & 1u;
                if (!mbar_wait(smem_u32(&tail->accum_empty[buf]), bph ^ 1u, status, kStatusTimeoutAccum)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>((buf * C::kIssuers + j) * kBN);
                int sl = 0;  // stage within the tile
                for (int kb = 0; kb < kb_n; kb += C::kBlocks, ++i, ++sl) {
                    if (sl % C::kIssuers != j) continue;
                    const int as = static_cast<int>(i % C::kASlots);
                    const int xs = static_cast<int>(i % C::kActStages);
                    if (!mbar_wait(smem_u32(&tail->afull[as]), (i / C::kASlots) & 1u, status, kStatusTimeoutFull) ||
                        !mbar_wait(smem_u32(&tail->xfull[xs]), (i / C::kActStages) & 1u, status,
                                   kStatusTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nblk = min(C::kBlocks, kb_n - kb);
                    for (int b = 0; b < nblk; ++b) {
                        const uint32_t b_base = smem_u32(act_ring + xs * C::kBBytes + b * kBN * 128);
                        const uint32_t a_tmem =
                            tmem_base + static_cast<uint32_t>(C::kAccCols + as * C::kSlotCols + b * 32);
#pragma unroll
                        for (int kk = 0; kk < kW16K / 16; ++kk) {
                            // B: K-major, 128-byte swizzle; K by 16 = 32 bytes inside the swizzle row.
                            const uint64_t bdesc = make_smem_desc(b_base + kk * 32, 16, 1024, 2);
                            tc_mma_f16_tmem_a(d_tmem, a_tmem + kk * 8, bdesc, idesc,
                                              (sl != j || b != 0 || kk != 0) ? 1u : 0u);
                        }
                    }
                    tc_commit(smem_u32(&tail->aempty[as]));
                    tc_commit(smem_u32(&tail->xempty[xs]));
                }
                if (ok) tc_commit(smem_u32(&tail->accum_full[buf]));
            }
            tc_commit(smem_u32(&tail->done));
            mbar_wait(smem_u32(&tail->done), 0, status, kStatusTimeoutDrain);
        }
    } else if (warp >= 4) {
        // ---------------- decoders ----------------
        const int q = warp & 3;
        const uint32_t group = static_cast<uint32_t>(warp - 4) >> 2;  // stages i with i % kDecGroups == group
        const int p = q * 32 + lane;  // packed column = TMEM lane
        uint32_t i = 0;
        bool ok = true;
        for (int t = first; t < total_tiles && ok; t += stride) {
            for (int kb = 0; kb < kb_n; kb += C::kBlocks, ++i) {
                if (i % kDecGroups != group) continue;
                const int ws = static_cast<int>(i % C::kWStages);
                const int as = static_cast<int>(i % C::kASlots);
                if (!mbar_wait(smem_u32(&tail->wfull[ws]), (i / C::kWStages) & 1u, status, kStatusTimeoutFull) ||
                    !mbar_wait(smem_u32(&tail->aempty[as]), ((i / C::kASlots) & 1u) ^ 1u, status,
                               kStatusTimeoutEmpty)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nblk = min(C::kBlocks, kb_n - kb);
                for (int b = 0; b < nblk; ++b) {
                    const uint8_t* blk = w_ring + ws * C::kWStageBytes + b * kW16BlockBytes;
                    const uint4 u0 = *reinterpret_cast<const uint4*>(blk + p * 16);
                    const uint4 u1 = *reinterpret_cast<const uint4*>(blk + 2048 + p * 16);
                    const uint32_t sw = *reinterpret_cast<const uint32_t*>(blk + kW16CodeBytes + p * 4);
                    const uint32_t s0 = scale_pair(sw), s1 = scale_pair(sw >> 8), s2 = scale_pair(sw >> 16),
                                   s3 = scale_pair(sw >> 24);
                    uint32_t r[32];
                    decode_word(u0.x, s0, r + 0);
                    decode_word(u0.y, s0, r + 4);
                    decode_word(u0.z, s1, r + 8);
                    decode_word(u0.w, s1, r + 12);
                    decode_word(u1.x, s2, r + 16);
                    decode_word(u1.y, s2, r + 20);
                    decode_word(u1.z, s3, r + 24);
                    decode_word(u1.w, s3, r + 28);
                    tmem_st_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                           static_cast<uint32_t>(C::kAccCols + as * C::kSlotCols + b * 32),
                                       r);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(smem_u32(&tail->afull[as]));
                    mbar_arrive(smem_u32(&tail->wempty[ws]));
                }
            }
        }
    } else {
        // ---------------- epilogue (warps 0..3) ----------------
        const int q = warp;
        uint16_t* out = static_cast<uint16_t*>(args.out);
        // the second issuer's accumulator holds a partial sum only if the tiles
        // have more than one stage
        const bool second = C::kIssuers > 1 && kb_n > C::kBlocks;
        int local = 0;
        for (int t = first; t < total_tiles; t += stride, ++local) {
            const W16Tile ti = w16_tile(t, tail->off, tail->mblk, n, args.n_tiles, kBN);
            const int buf = local & 1;
            const uint32_t bph = static_cast<uint32_t>(local >> 1) & 1u;
            const bool got = epi_all(mbar_wait(smem_u32(&tail->accum_full[buf]), bph, status, kStatusTimeoutAccum));
            if (!got) break;  // all four warps together
            tc_fence_after();
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(buf * C::kIssuers * kBN);
            const int valid = ti.rows;
            if (kSwiGLU) {
                const float sa = __ldg(args.mscale0 + ti.e) * 256.f;
                const float sb = __ldg(args.mscale1 + ti.e) * 256.f;
                if (q >= 2) {
#pragma unroll 1
                    for (int c0 = 0; c0 < kBN; c0 += 32) {
                        uint32_t b[32];
                        ld_acc<C::kIssuers, kBN>(tbase + c0, b, second);
#pragma unroll
                        for (int k = 0; k < 32; ++k)
                            xbuf[(c0 + k) * 64 + (q - 2) * 32 + lane] = __uint_as_float(b[k]) * sb;
                    }
                }
                epi_bar();
                if (q < 2) {
                    const int col = ti.j * 64 + q * 32 + lane;
#pragma unroll 1
                    for (int c0 = 0; c0 < kBN; c0 += 32) {
                        uint32_t a[32];
                        ld_acc<C::kIssuers, kBN>(tbase + c0, a, second);
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const float h = silu_w16(__uint_as_float(a[k]) * sa) * xbuf[(c0 + k) * 64 + q * 32 + lane];
                            if (c0 + k < valid)
                                out[(static_cast<int64_t>(ti.row0) + c0 + k) * args.out_cols + col] =
                                    __bfloat16_as_ushort(__float2bfloat16_rn(h));
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&tail->accum_empty[buf]));
                epi_bar();  // xbuf is free for the next tile
            } else {
                const float so = __ldg(args.mscale0 + ti.e) * 256.f;
                const int col = ti.j * kW16Cols + q * 32 + lane;
#pragma unroll 1
                for (int c0 = 0; c0 < kBN; c0 += 32) {
                    uint32_t a[32];
                    ld_acc<C::kIssuers, kBN>(tbase + c0, a, second);
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if (c0 + k < valid)
                            out[(static_cast<int64_t>(ti.row0) + c0 + k) * args.out_cols + col] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(a[k]) * so));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&tail->accum_empty[buf]));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    griddep_launch_dependents();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// Fields of an E2M1 code (bit 0 mantissa, bits 1-2 exponent, bit 3 sign) go
// to these bf16 bit positions of the lower half (the upper half: + 16).
__device__ __forceinline__ int w16_target(int field) { return field == 3 ? 15 : 6 + field; }

// Rotation that brings pair i's field back to its bf16 position.
__device__ __forceinline__ int w16_rotation(int pair, int field) {
    if (pair == 3) return field == 0 ? 14 : 6;
    return pair == 0 ? 0 : (pair == 1 ? 4 : 10);
}

// Thread = (expert, tile, 64-row step, packed column): one column's 64 codes
// of the step as 8 words, and its 4 block scales.
__global__ void __launch_bounds__(256)
    w4a16_pack_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ bscale,
                      const uint8_t* __restrict__ codes_pair, const uint8_t* __restrict__ bscale_pair, int K, int N,
                      int n_tiles, uint8_t* __restrict__ out) {
    const int steps = K / kW16K;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (item >= static_cast<int64_t>(n_tiles) * steps * kW16Cols) return;
    const int e = blockIdx.y;
    const int p = static_cast<int>(item % kW16Cols);
    const int64_t rest = item / kW16Cols;
    const int s = static_cast<int>(rest % steps);
    const int j = static_cast<int>(rest / steps);
    const uint8_t* src = codes;
    const uint8_t* ssrc = bscale;
    int col;
    if (codes_pair) {
        col = j * 64 + (p & 63);
        if (p >= 64) {
            src = codes_pair;
            ssrc = bscale_pair;
        }
    } else {
        col = j * kW16Cols + p;
    }
    const int64_t half_cols = N / 2;
    uint32_t words[8];
#pragma unroll 1
    for (int wd = 0; wd < 8; ++wd) {
        uint32_t w = 0;
        for (int r = 0; r < 8; ++r) {
            const int64_t k = static_cast<int64_t>(s) * kW16K + wd * 8 + r;
            const uint32_t byte = src[(static_cast<int64_t>(e) * K + k) * half_cols + col / 2];
            const uint32_t code = (byte >> (4 * (col & 1))) & 0xFu;
            const int pair = r >> 1, hi = r & 1;
            for (int f = 0; f < 4; ++f) {
                const int pos = (w16_target(f) + 16 * hi + w16_rotation(pair, f)) & 31;
                w |= ((code >> f) & 1u) << pos;
            }
        }
        words[wd] = w;
    }
    uint8_t* blk = out + ((static_cast<int64_t>(e) * n_tiles + j) * steps + s) * kW16BlockBytes;
    *reinterpret_cast<uint4*>(blk + p * 16) = make_uint4(words[0], words[1], words[2], words[3]);
    *reinterpret_cast<uint4*>(blk + 2048 + p * 16) = make_uint4(words[4], words[5], words[6], words[7]);
    uint32_t sc = 0;
    for (int g = 0; g < 4; ++g)
        sc |= static_cast<uint32_t>(ssrc[(static_cast<int64_t>(e) * (K / 16) + 4 * s + g) * N + col]) << (8 * g);
    *reinterpret_cast<uint32_t*>(blk + kW16CodeBytes + p * 4) = sc;
}

template <bool kSwiGLU, int kBN>
cudaError_t launch_w16(const CUtensorMap& tm, const W4a16GemmArgs& a, int num_sms, cudaStream_t st) {
    constexpr int smem = w16_smem_bytes<kBN>();
    cudaError_t e = cudaFuncSetAttribute(w4a16_gemm_kernel<kSwiGLU, kBN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int64_t max_tiles = ((a.R + kBN - 1) / kBN + a.n) * static_cast<int64_t>(a.n_tiles);
    int64_t g = num_sms;
    if (max_tiles < g) g = max_tiles;
    if (g < 1) g = 1;
    launch_k(w4a16_gemm_kernel<kSwiGLU, kBN>, dim3(static_cast<unsigned>(g)), dim3(W16Cfg<kBN>::kThreads), smem, st, tm,
             a);
    return cudaGetLastError();
}

}  // namespace

int w4a16_tile_rows(int64_t R, int n) { return R <= 32 * static_cast<int64_t>(n) ? 32 : 128; }

cudaError_t launch_w4a16_pack(const uint8_t* codes, const uint8_t* bscale, const uint8_t* codes_pair,
                              const uint8_t* bscale_pair, int n, int K, int N, uint8_t* packed, cudaStream_t st) {
    const int n_tiles = codes_pair ? N / 64 : N / kW16Cols;
    const int64_t items = static_cast<int64_t>(n_tiles) * (K / kW16K) * kW16Cols;
    const dim3 grid(static_cast<unsigned>((items + 255) / 256), static_cast<unsigned>(n));
    w4a16_pack_kernel<<<grid, 256, 0, st>>>(codes, bscale, codes_pair, bscale_pair, K, N, n_tiles, packed);
    return cudaGetLastError();
}

cudaError_t launch_w4a16_gemm1(const CUtensorMap& tm_xp, const W4a16GemmArgs& a, int tile_rows, int num_sms,
                               cudaStream_t st) {
    return tile_rows == 32 ? launch_w16<true, 32>(tm_xp, a, num_sms, st)
                           : launch_w16<true, 128>(tm_xp, a, num_sms, st);
}

cudaError_t launch_w4a16_gemm2(const CUtensorMap& tm_h, const W4a16GemmArgs& a, int tile_rows, int num_sms,
                               cudaStream_t st) {
    return tile_rows == 32 ? launch_w16<false, 32>(tm_h, a, num_sms, st)
                           : launch_w16<false, 128>(tm_h, a, num_sms, st);
}

}  // namespace moe
