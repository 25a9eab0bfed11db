// gemv.cuh - block-quantized GEMV for sm_100a (batch 1) on the GGUF-style
// layouts (the tiled layouts take integer dots, qmma.cuh), with optional fused
// prologue (RMSNorm of the input) and epilogues (residual add, SwiGLU of a
// gate/up row pair, RoPE + fp16 KV-cache append for a fused QKV projection).
//
// The GEMV kernel of the ntransformer news summary ("Arquitectura y estructura
// del código": cuda/ holds GEMV, RMSNorm, RoPE, SwiGLU and softmax kernels),
// redesigned for B200: batch-1 GEMV is a pure weight stream, so the kernel is
// built to keep HBM busy, not to use tensor cores.
//
// Structure (one CTA per SM, 8 consumer warps + 1 producer warp):
//  * The CTA owns a contiguous range of output rows.  A stage holds 8 row slots
//    x one chunk of CE columns of each row (CE = 256 threads x E elements).  The
//    producer warp streams stages with 1-D bulk copies (cp.async.bulk, L2
//    evict-first) into a ring of shared-memory stages guarded by mbarriers.
//  * The input vector is staged once per CTA into shared memory, pre-scaled and
//    laid out so each consumer thread reads its E values as conflict-free
//    16-byte loads; each value read is reused for the 8 rows of a stage.
//  * Dequantization happens in registers: a code field is masked straight into
//    the bit pattern of an fp32 number below 2^-125 (exact value code * 2^(p-149)
//    for a field at bit p), so one logic op turns a code into a float and the
//    dot products run as paired fp32 FMAs (fma.rn.f32x2).  The input is
//    pre-multiplied by 2^(S-p) so every product is code * x * 2^(S-149); the
//    format's code offset (128, 8, 32 or the Q4_K min) is removed per block with
//    the same products taken on the offset, and the row total is scaled back by
//    2^(149-S).  All scalings are exact powers of two.
//  * Row totals are reduced warp-wise (transposed butterfly, 9 shuffles for 8
//    rows) and across warps through shared memory, then the epilogue runs.
#pragma once

#include "common.cuh"

namespace ntx {
namespace gemv {

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kOwners = 256;           // element owners per chunk (consumer threads per group)
constexpr int kHeader = 2048;          // barriers + reduction scratch at the start of shared memory
constexpr int kMaxStages = 8;
constexpr int kSmemLimit = 227 * 1024;
constexpr uint32_t kWaitPolls = 1u << 22;   // bounded mbarrier waits (far above any real stage time)

enum Epi { EPI_STORE = 0, EPI_ADD = 1, EPI_SWIGLU = 2, EPI_QKV = 3 };
enum Pro { PRO_X = 0, PRO_RMSNORM = 1 };

struct Params {
    const uint8_t* W;     // packed rows (gate rows for SwiGLU)
    const uint8_t* W2;    // up rows for SwiGLU
    int64_t row_bytes;
    int M;                // output rows
    int K;                // columns
    const float* x;       // input (PRO_X) or the vector to normalise (PRO_RMSNORM)
    const float* norm_w;  // RMSNorm weights
    float eps;
    float* y;             // output (EPI_STORE / EPI_ADD / EPI_SWIGLU)
    // EPI_QKV
    int q_rows, kv_rows, head_dim, max_ctx;
    const int32_t* pos_dev;
    int32_t pos;
    const float* rope_cs; // [head_dim / 2][cos, sin] of pos theta^(-2i/head_dim), written before the kernel
    __half* k_cache;
    __half* v_cache;
    float* q_out;
    // launch shape
    int n_stages;
    int n_chunks;
    int chunk_elems;      // CE
    int chunk_bytes;      // bytes of a full chunk of one row
    int stage_bytes;
    int x_bytes;
    int use_pdl;
    int recv_bytes;       // tiled GEMV: bytes of the per-group row sums of a CTA pair
    int fs_off;           // tiled GEMV: byte offset of the per-step factors from the x words
    int stall_stage;      // tiled GEMV, tests of the bounded waits: the producer issues no copy
                          // from this stage on, so the consumers' wait for it runs out (-1: off)
    // multiplier that lets a shift run as an integer multiply on the FMA pipe
    // (v >> 8 == umulhi(v, 2^24)); passed in so it stays a multiply
    uint32_t m24;
};

// The vectors of one multi-vector tiled GEMV launch (entries v < the launch's count are
// used): y_v = W x_v with the same fused prologue and epilogue for every v.
constexpr int kMaxVecs = 4;
struct Vecs {
    const float* x[kMaxVecs];          // input, or the vector to normalise (PRO_RMSNORM)
    float* y[kMaxVecs];                // output (EPI_STORE / EPI_ADD / EPI_SWIGLU)
    float* q_out[kMaxVecs];            // EPI_QKV: q
    const int32_t* pos_dev[kMaxVecs];  // EPI_QKV: the vector's position
    const float* rope_cs[kMaxVecs];    // EPI_QKV: [head_dim / 2][cos, sin] of that position
};

template <int QT>
struct Fmt;

// Row slots per stage: 16 for the formats whose threads own 16 elements, 8 for
// the 32-element ones; each of the two consumer groups takes half of the slots.
// (Measured on B200: more rows per thread per stage beats a deeper ring of smaller
// stages, because the per-row and per-stage costs of the consumers dominate.)
template <int QT>
struct Slots {
    static constexpr int value = ((QT & 3) == NTX_Q8_0 || (QT & 3) == NTX_Q4_0) ? 16 : 8;
    static constexpr int per_thread = value / 2;
};

// Elements per consumer thread per row chunk, and positions of the code fields.
template <>
struct Fmt<NTX_Q8_0> {
    static constexpr int E = 16, BE = 32, BB = 34;
};
template <>
struct Fmt<NTX_Q4_0> {
    static constexpr int E = 16, BE = 32, BB = 18;
};
template <>
struct Fmt<NTX_Q4_K> {
    static constexpr int E = 32, BE = 256, BB = 144;
};
template <>
struct Fmt<NTX_Q6_K> {
    static constexpr int E = 32, BE = 256, BB = 210;
};

// ------------------------------------------------------------------ element maps
// chunk-local element index and code-field bit position of value (piece j, lane k)
// of consumer thread t.  Pieces are groups of 4 consecutive values.

__device__ __forceinline__ int pos_of_byte(int k) { return k < 3 ? 8 * k : 16; }

template <int QT>
__device__ __forceinline__ void elem_of(int t, int j, int k, int& e, int& p);

template <>
__device__ __forceinline__ void elem_of<NTX_Q8_0>(int t, int j, int k, int& e, int& p)
{
    // thread t: half `t & 1` of block t >> 1; code word j holds elements 16t+4j..+3
    e = 16 * t + 4 * j + k;
    p = pos_of_byte(k);
}

template <>
__device__ __forceinline__ void elem_of<NTX_Q4_0>(int t, int j, int k, int& e, int& p)
{
    // thread t: code bytes 8h..8h+7 of block b (h = t & 1, b = t >> 1); piece j:
    // word j & 1, low nibbles (j < 2) = elements 8h+4w+k, high nibbles = 16+8h+4w+k
    const int b = t >> 1, h = t & 1, w = j & 1, hi = j >> 1;
    e = 32 * b + 16 * hi + 8 * h + 4 * w + k;
    p = 4 * hi + pos_of_byte(k);
}

template <>
__device__ __forceinline__ void elem_of<NTX_Q4_K>(int t, int j, int k, int& e, int& p)
{
    // thread t: superblock t >> 3, 64-element group c = (t & 7) >> 1, code bytes
    // 32c + 16h .. +15 (h = t & 1) = 4 words; piece j < 4: low nibbles of word j
    // (elements 64c + 16h + 4j + k, sub-block 2c); j >= 4: high nibbles of word j-4
    // (elements 64c + 32 + 16h + 4(j-4) + k, sub-block 2c+1)
    const int sb = t >> 3, c = (t & 7) >> 1, h = t & 1, hi = j >> 2, w = j & 3;
    e = 256 * sb + 64 * c + 32 * hi + 16 * h + 4 * w + k;
    p = 4 * hi + pos_of_byte(k);
}

template <>
__device__ __forceinline__ void elem_of<NTX_Q6_K>(int t, int j, int k, int& e, int& p)
{
    // thread t: superblock t >> 3, half hh = (t & 7) >> 2, columns l in
    // 8u .. 8u+7 (u = t & 3); piece j = 2 qq + w: elements 128hh + 32qq + 8u + 4w + k
    const int sb = t >> 3, hh = (t & 7) >> 2, u = t & 3, qq = j >> 1, w = j & 1;
    e = 256 * sb + 128 * hh + 32 * qq + 8 * u + 4 * w + k;
    p = pos_of_byte(k);
}

// Blocks (or superblocks) of a chunk row that thread t reads; used to skip
// threads past the end of a partial chunk.
template <int QT>
__device__ __forceinline__ int block_of_thread(int t)
{
    return (QT == NTX_Q8_0 || QT == NTX_Q4_0) ? (t >> 1) : (t >> 3);
}

// ------------------------------------------------------------------ per-row dot

// fp32 number whose bit pattern is the integer v (< 2^24): value v * 2^-149.
__device__ __forceinline__ uint32_t as_tiny(uint32_t v) { return v; }

// Returns, in units of 2^(S-149): sum over this thread's elements of the
// dequantized weight (without the fp16 d) times x, with d folded in per block.
template <int QT>
struct Dot;

template <>
struct Dot<NTX_Q8_0> {
    // x: 8 pairs (4 pieces x 2), off: sum of 128 * x'' over the 16 elements (tiny units)
    static __device__ __forceinline__ float row(const uint8_t* row, int t, const uint64_t (&x)[8], float off)
    {
        const int boff = 34 * (t >> 1);
        const float d = f16_bits_to_f32(*reinterpret_cast<const uint16_t*>(row + boff));
        const int coff = boff + 2 + 16 * (t & 1);
        const uint32_t* base = reinterpret_cast<const uint32_t*>(row + (coff & ~3));
        const uint32_t sh = (coff & 3) * 8;
        uint32_t raw[5];
#pragma unroll
        for (int i = 0; i < 5; ++i) raw[i] = base[i];
        uint64_t a0 = 0, a1 = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t w = __funnelshift_r(raw[j], raw[j + 1], sh) ^ 0x80808080u;
            fma2(a0, pack2(w & 0xFFu, w & 0xFF00u), x[2 * j]);
            fma2(a1, pack2(w & 0xFF0000u, (w >> 8) & 0xFF0000u), x[2 * j + 1]);
        }
        const f2 s0 = f2_from(a0), s1 = f2_from(a1);
        return d * (((s0.x + s0.y) + (s1.x + s1.y)) - off);
    }
};

template <>
struct Dot<NTX_Q4_0> {
    static __device__ __forceinline__ float row(const uint8_t* row, int t, const uint64_t (&x)[8], float off)
    {
        const int boff = 18 * (t >> 1);
        const float d = f16_bits_to_f32(*reinterpret_cast<const uint16_t*>(row + boff));
        const int coff = boff + 2 + 8 * (t & 1);
        const uint32_t* base = reinterpret_cast<const uint32_t*>(row + (coff & ~3));
        const uint32_t sh = (coff & 3) * 8;
        const uint32_t r0 = base[0], r1 = base[1], r2 = base[2];
        const uint32_t w0 = __funnelshift_r(r0, r1, sh), w1 = __funnelshift_r(r1, r2, sh);
        uint64_t a0 = 0, a1 = 0;
        // piece j = 2 hi + w: pairs x[2j], x[2j+1]
        {
            const uint32_t v = w0, v8 = w0 >> 8;
            fma2(a0, pack2(v & 0xFu, v & 0xF00u), x[0]);
            fma2(a1, pack2(v & 0xF0000u, v8 & 0xF0000u), x[1]);
            fma2(a0, pack2(v & 0xF0u, v & 0xF000u), x[4]);
            fma2(a1, pack2(v & 0xF00000u, v8 & 0xF00000u), x[5]);
        }
        {
            const uint32_t v = w1, v8 = w1 >> 8;
            fma2(a0, pack2(v & 0xFu, v & 0xF00u), x[2]);
            fma2(a1, pack2(v & 0xF0000u, v8 & 0xF0000u), x[3]);
            fma2(a0, pack2(v & 0xF0u, v & 0xF000u), x[6]);
            fma2(a1, pack2(v & 0xF00000u, v8 & 0xF00000u), x[7]);
        }
        const f2 s0 = f2_from(a0), s1 = f2_from(a1);
        return d * (((s0.x + s0.y) + (s1.x + s1.y)) - off);
    }
};

template <>
struct Dot<NTX_Q4_K> {
    // x: 16 pairs (8 pieces); xs_lo / xs_hi: sum of x'' * 2^p for the low / high
    // nibble elements (tiny units), for the min terms.
    static __device__ __forceinline__ float row(const uint8_t* row, int t, const uint64_t (&x)[16], float xs_lo,
                                                float xs_hi, uint32_t m24)
    {
        const int sbo = 144 * (t >> 3);
        const int c = (t & 7) >> 1, h = t & 1;
        const uint4 hdr = *reinterpret_cast<const uint4*>(row + sbo);   // d | dmin, s0, s1, s2
        const uint4 q = *reinterpret_cast<const uint4*>(row + sbo + 16 + 32 * c + 16 * h);
        const float d = f16_bits_to_f32((uint16_t)(hdr.x & 0xFFFF));
        const float dmin = f16_bits_to_f32((uint16_t)(hdr.x >> 16));
        // scale / min of sub-blocks 2c (A) and 2c+1 (B)
        uint32_t scA, scB, mA, mB;
        if (c < 2) {
            const int jA = 2 * c, jB = 2 * c + 1;
            scA = (hdr.y >> (8 * jA)) & 63u;
            scB = (hdr.y >> (8 * jB)) & 63u;
            mA = (hdr.z >> (8 * jA)) & 63u;
            mB = (hdr.z >> (8 * jB)) & 63u;
        } else {
            const int jA = 2 * c - 4, jB = 2 * c - 3;
            scA = ((hdr.w >> (8 * jA)) & 15u) | (((hdr.y >> (8 * jA + 6)) & 3u) << 4);
            scB = ((hdr.w >> (8 * jB)) & 15u) | (((hdr.y >> (8 * jB + 6)) & 3u) << 4);
            mA = ((hdr.w >> (8 * jA + 4)) & 15u) | (((hdr.z >> (8 * jA + 6)) & 3u) << 4);
            mB = ((hdr.w >> (8 * jB + 4)) & 15u) | (((hdr.z >> (8 * jB + 6)) & 3u) << 4);
        }
        uint64_t lo0 = 0, lo1 = 0, hi0 = 0, hi1 = 0;
        const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const uint32_t v = qw[w], v8 = __umulhi(v, m24);
            fma2(lo0, pack2(v & 0xFu, v & 0xF00u), x[2 * w]);
            fma2(lo1, pack2(v & 0xF0000u, v8 & 0xF0000u), x[2 * w + 1]);
            fma2(hi0, pack2(v & 0xF0u, v & 0xF000u), x[8 + 2 * w]);
            fma2(hi1, pack2(v & 0xF00000u, v8 & 0xF00000u), x[8 + 2 * w + 1]);
        }
        const f2 l0 = f2_from(lo0), l1 = f2_from(lo1), g0 = f2_from(hi0), g1 = f2_from(hi1);
        const float sA = (l0.x + l0.y) + (l1.x + l1.y);
        const float sB = (g0.x + g0.y) + (g1.x + g1.y);
        const float dA = d * (float)scA, dB = d * (float)scB;
        const float mnA = dmin * (float)mA, mnB = dmin * (float)mB;
        return (dA * sA + dB * sB) - (mnA * xs_lo + mnB * xs_hi);
    }
};

template <>
struct Dot<NTX_Q6_K> {
    // x: 16 pairs (8 pieces, piece j = 2 qq + w); off[qq]: sum of 32 * x'' * 2^p over the
    // 8 elements of group qq (tiny units).
    static __device__ __forceinline__ float row(const uint8_t* row, int t, const uint64_t (&x)[16],
                                                const float (&off)[4])
    {
        const int sbo = 210 * (t >> 3);
        const int hh = (t & 7) >> 2, u = t & 3;
        const uint32_t sh = (sbo & 3) * 8;          // superblock starts are 2-byte aligned
        const uint8_t* sb = row + (sbo & ~3);       // 4-byte aligned base, content shifted by sh
        const int a_ql = 64 * hh + 8 * u;           // ql bytes of qq = 0, 2 (8 bytes)
        const int b_ql = 64 * hh + 32 + 8 * u;      // ql bytes of qq = 1, 3
        const int c_qh = 128 + 32 * hh + 8 * u;     // qh bytes (8 bytes)
        const int s_sc = 192 + 8 * hh;              // scales 8hh .. 8hh+7
        auto words2 = [&](int o, uint32_t& lo, uint32_t& hi) {
            const uint32_t* p = reinterpret_cast<const uint32_t*>(sb + o);
            const uint32_t r0 = p[0], r1 = p[1], r2 = p[2];
            lo = __funnelshift_r(r0, r1, sh);
            hi = __funnelshift_r(r1, r2, sh);
        };
        uint32_t qa0, qa1, qb0, qb1, qh0, qh1, sc0, sc1;
        words2(a_ql, qa0, qa1);
        words2(b_ql, qb0, qb1);
        words2(c_qh, qh0, qh1);
        words2(s_sc, sc0, sc1);
        const float d = f16_bits_to_f32(*reinterpret_cast<const uint16_t*>(row + sbo + 208));
        // sub-block of group qq: 8hh + 2qq + (u >> 1); its scale is byte 2qq + (u >> 1) of sc0:sc1
        const int su = u >> 1;
        float ds[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            const int byte = 2 * qq + su;
            const uint32_t word = byte < 4 ? sc0 : sc1;
            const int8_t s = (int8_t)((word >> (8 * (byte & 3))) & 0xFF);
            ds[qq] = d * (float)s;
        }
        float res = 0.f;
        const uint32_t qa[2] = {qa0, qa1}, qb[2] = {qb0, qb1}, qh[2] = {qh0, qh1};
        uint64_t acc[4][2];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) acc[qq][0] = acc[qq][1] = 0;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            const uint32_t hA = qh[w] & 0x33333333u;           // high bits of qq 0 (bits 0-1) and 2 (bits 4-5)
            const uint32_t hB = (qh[w] >> 2) & 0x33333333u;    // high bits of qq 1 and 3
            uint32_t code[4];
            // code byte = low nibble | high 2 bits << 4 (bits 6-7 stay zero)
            code[0] = (qa[w] & 0x0F0F0F0Fu) | ((hA << 4) & 0xF0F0F0F0u);
            code[1] = (qb[w] & 0x0F0F0F0Fu) | ((hB << 4) & 0xF0F0F0F0u);
            code[2] = ((qa[w] >> 4) & 0x0F0F0F0Fu) | (hA & 0xF0F0F0F0u);
            code[3] = ((qb[w] >> 4) & 0x0F0F0F0Fu) | (hB & 0xF0F0F0F0u);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const uint32_t v = code[qq];
                fma2(acc[qq][0], pack2(v & 0xFFu, v & 0xFF00u), x[2 * (2 * qq + w)]);
                fma2(acc[qq][1], pack2(v & 0xFF0000u, (v >> 8) & 0xFF0000u), x[2 * (2 * qq + w) + 1]);
            }
        }
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            const f2 a = f2_from(acc[qq][0]), b = f2_from(acc[qq][1]);
            res = fmaf(ds[qq], ((a.x + a.y) + (b.x + b.y)) - off[qq], res);
        }
        return res;
    }
};


// One row of one stage for this thread, in units of 2^(S-149).
template <int QT>
__device__ __forceinline__ float dot_row(const uint8_t* row, int lt, const uint64_t (&xr)[2 * (Fmt<QT>::E / 4)],
                                         const float (&offs)[4], const Params& P)
{
    if constexpr (QT == NTX_Q8_0) {
        return Dot<NTX_Q8_0>::row(row, lt, xr, offs[0]);
    } else if constexpr (QT == NTX_Q4_0) {
        return Dot<NTX_Q4_0>::row(row, lt, xr, offs[0]);
    } else if constexpr (QT == NTX_Q4_K) {
        return Dot<NTX_Q4_K>::row(row, lt, xr, offs[0], offs[1], P.m24);
    } else {
        return Dot<NTX_Q6_K>::row(row, lt, xr, offs);
    }
}

// ------------------------------------------------------------------ helpers

// x * 2^e for |e| <= 252, exact (two power-of-two multiplies).
__device__ __forceinline__ float scale2(float v, int e)
{
    int e1 = e / 2, e2 = e - e1;
    return v * __uint_as_float((uint32_t)(127 + e1) << 23) * __uint_as_float((uint32_t)(127 + e2) << 23);
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Reduce v over the 256 consumer threads (result in every consumer thread).
__device__ __forceinline__ float consumers_reduce(float v, float* red, bool is_max)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    v = is_max ? warp_max(v) : warp_sum(v);
    if (lane == 0) red[warp] = v;
    named_bar_sync(1, kConsumers);
    float r = red[0];
#pragma unroll
    for (int w = 1; w < kConsumerWarps; ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
    named_bar_sync(1, kConsumers);
    return r;
}

}  // namespace gemv
}  // namespace ntx
