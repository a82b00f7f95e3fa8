// On-the-fly transposition of a 4-bit operand tile in shared memory.
//
// FourTune section 3.2 ("4-Bit Backward Pass via Block-Quantization", and the on-the-fly
// transposition named in section 1): the backward's dX GEMM multiplies by Q(R)^T,
// whose K-major layout is the transpose of the stored Q(R).  Instead of keeping a second
// copy of the codes (half a byte per weight), the GEMM's producer loads the untransposed
// tile of Q(R) into the B operand slot and the CTA's four scale warps rewrite it in place
// into the K-major, 128-byte-swizzled layout the MMA reads.  The scale factors of the
// transposed operand are unchanged (the 16 x 16 block scale grid, transposed).
//
// Cost.  The rewrite is about five integer operations per 32-bit word (the byte moves by
// byte permutes, the nibble moves by shift-and-select), and the four scale warps run on
// the four SM sub-partitions, so it is bound by the sub-partitions' integer pipes; it
// lengthens the scale warps' per-stage chain beyond the MMAs' 512 cycles.
//
// Geometry.  The raw tile holds 256 rows n (the GEMM's reduction index) of RB bytes, i.e.
// 2 RB output columns with two codes per byte, the even column in the low nibble, as TMA
// writes it with the 64-byte swizzle (RB = 64) or the 128-byte swizzle (RB = 128).  The
// transposed tile holds 2 RB rows (output columns) of 128 bytes: row r, byte x holds the
// codes of reduction rows 2x (low nibble) and 2x + 1, 16-byte chunk c of row r stored at
// chunk c ^ (r % 8) (the 128-byte swizzle).
//
// Work split.  The tile is cut into 8 x 8 blocks of codes: raw rows 8w .. 8w+7 (w < 32)
// by output columns 8kb .. 8kb+7, i.e. one 32-bit word of each of eight raw rows, which
// becomes one 32-bit word (word w) of each of eight transposed rows.  Lane l of scale warp
// q takes w4 = l % 8 and kbl = l / 8; for each 16-byte chunk c = q + 4h of the raw rows
// (h < RB / 64) it handles kb = 4c + kbl and the four blocks w = 4 w4 + bi (bi < 4), so its
// eight transposed rows get one 16-byte store each (words 4 w4 .. 4 w4 + 3).
//
// Banks.  Lane l reads row j of its blocks at load step j ^ w4 rather than at step j: with
// that rotation the 32 lanes hit 32 different banks at every load, and at every 16-byte
// store the eight lanes of each quarter warp hit eight different bank groups.  The
// transposition undoes the rotation for free: its three exchange stages pair rows at
// distance 4, 2 and 1, and the rotation only decides which of the two registers holds the
// lower row of a pair: a byte-permute selector in the first two stages, a select in the
// last.
#pragma once
#include <cstdint>

namespace ft {
namespace xpose {

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// Bytes of the 8-byte value {b, a} (a = bytes 0-3) picked by the four selector nibbles.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

template <int RB>
struct Regs {
    static_assert(RB == 64 || RB == 128, "raw rows of 64 or 128 bytes");
    static constexpr int H = RB / 64;  // 16-byte chunks per lane
    uint32_t v[H][4][8];               // [chunk][block][row slot]
};

// Phase 1: this lane's words of the raw tile into registers.  Slot j of block bi holds raw
// row 32 w4 + 8 bi + (j ^ w4), word kb of that row.
template <int RB>
__device__ __forceinline__ void load(uint32_t tile, int q, int lane, Regs<RB>& r) {
    const int w4 = lane & 7, kbl = lane >> 3;
#pragma unroll
    for (int h = 0; h < Regs<RB>::H; ++h) {
        const int c = q + 4 * h;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int jr = j ^ w4;
            const int sw = RB == 64 ? ((jr >> 1) & 3) : jr;  // swizzle phase of the raw row
            const uint32_t a = tile + w4 * (32 * RB) + jr * RB + ((c ^ sw) << 4) + (kbl << 2);
#pragma unroll
            for (int bi = 0; bi < 4; ++bi) r.v[h][bi][j] = lds32(a + bi * (8 * RB));
        }
    }
}

// Transposes one 8 x 8 block of 4-bit codes whose row slots are rotated by `rot` (slot j
// holds row j ^ rot).  On return, v[p] holds transposed row p: nibble j = code (j, p).
__device__ __forceinline__ void block8(uint32_t (&v)[8], int rot) {
    // distance 4: 4 x 4 quadrants; upper/lower half-words trade places
    const uint32_t s1a = (rot & 4) ? 0x1054u : 0x5410u, s1b = (rot & 4) ? 0x3276u : 0x7632u;
    // distance 2: 2 x 2 sub-blocks; bytes trade places
    const uint32_t s2a = (rot & 2) ? 0x2604u : 0x6240u, s2b = (rot & 2) ? 0x3715u : 0x7351u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t a = prmt(v[j], v[j + 4], s1a), b = prmt(v[j], v[j + 4], s1b);
        v[j] = a;
        v[j + 4] = b;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = (i & 1) + 4 * (i >> 1);  // 0, 1, 4, 5
        const uint32_t a = prmt(v[j], v[j + 2], s2a), b = prmt(v[j], v[j + 2], s2b);
        v[j] = a;
        v[j + 2] = b;
    }
    // distance 1: single codes; nibbles trade places
    const bool odd = (rot & 1) != 0;
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
        const uint32_t lo = odd ? v[j + 1] : v[j], hi = odd ? v[j] : v[j + 1];
        v[j] = (lo & 0x0F0F0F0Fu) | ((hi << 4) & 0xF0F0F0F0u);
        v[j + 1] = ((lo >> 4) & 0x0F0F0F0Fu) | (hi & 0xF0F0F0F0u);
    }
}

// Phase 2 arithmetic: every block of this lane, in registers.
template <int RB>
__device__ __forceinline__ void transpose(int lane, Regs<RB>& r) {
#pragma unroll
    for (int h = 0; h < Regs<RB>::H; ++h)
#pragma unroll
        for (int bi = 0; bi < 4; ++bi) block8(r.v[h][bi], lane & 7);
}

// Phase 2 stores: transposed row 8 kb + p, 16-byte chunk w4, at its swizzled place.  Every
// lane of every scale warp must have finished `load` first (the tile is rewritten in place).
template <int RB>
__device__ __forceinline__ void store(uint32_t tile, int q, int lane, const Regs<RB>& r) {
    const int w4 = lane & 7, kbl = lane >> 3;
#pragma unroll
    for (int h = 0; h < Regs<RB>::H; ++h) {
        // row 8 kb starts a 1024-byte swizzle atom; row 8 kb + p's chunk w4 sits at
        // +128 p + 16 (w4 ^ p), i.e. the atom address with 144 p xor-ed in
        const uint32_t row0 = tile + (4 * (q + 4 * h) + kbl) * 1024 + (w4 << 4);
#pragma unroll
        for (int p = 0; p < 8; ++p)
            sts128(row0 ^ static_cast<uint32_t>(p * 0x90), r.v[h][0][p], r.v[h][1][p], r.v[h][2][p], r.v[h][3][p]);
    }
}

}  // namespace xpose
}  // namespace ft
