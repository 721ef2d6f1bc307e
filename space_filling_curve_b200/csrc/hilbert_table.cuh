// hilbert_table.cuh -- the 3-D Hilbert index of a grid point (Tessera's
// space-filling-curve order; Skilling, "Programming the Hilbert curve",
// 2004) as a finite state machine over the levels of the point's Morton
// code, two levels per table lookup.
//
// Skilling's transform visits the levels from the top.  At level l it reads
// the level-l bits (a, b, c) of the current x, y, z and applies to every bit
// below l, in this order: invert x if a; then invert x if b, else exchange
// x and y; then invert x if c, else exchange x and z.  Each of these acts on
// every lower level the same way, so the transform that the levels above l
// have built up is one signed permutation T of the three bits of a level,
// and the bits the curve sees at level l are T(o) for the original octant
// o.  The final Gray code (y ^= x, z ^= y) is per level; its fold (every bit
// of a level XORed with the parity of z's Gray bits above it) is a running
// parity f.  So the state (T, f) and the octant o give the key's three bits
// at this level and the next state.  Of the 48 signed permutations x 2
// parities, 48 states are reachable from the identity.  The key interleaves
// the three transformed words most-significant level first, x's bit highest
// in each triple.
//
// The tables are built at compile time from those rules alone: each state
// is represented by T as an explicit map of the 8 octants.  Entry layout:
//   two[s * 64 + (o_hi << 3 | o_lo)] = digits (6 bits: level l's triple, then
//                                      level l-1's) | next state << 6
//   one[s * 8 + o]                   = digit (3 bits) | next state << 6
// with the identity and f = 0 as state 0.  Bit order of an octant and of a
// digit: x highest, z lowest (the Morton interleave of morton_key()).
#pragma once

#include <cstdint>

namespace tess {

constexpr int HT_MAX_STATES = 96;

struct alignas(16) HilbertTables {
    uint16_t two[HT_MAX_STATES * 64];
    uint16_t one[HT_MAX_STATES * 8];
    int nstates;
};

namespace hilbert_fsm {

// A state: T as the images of the 8 octants (3 bits each), and the parity.
struct State {
    uint32_t map;   // bits 3k..3k+2: T(k)
    uint32_t f;
};

constexpr uint32_t image(uint32_t map, uint32_t o) { return (map >> (3 * o)) & 7u; }

// Apply a bit operation g (on a level's 3 bits) after T.
constexpr uint32_t flip_x(uint32_t t) { return t ^ 4u; }
constexpr uint32_t swap_xy(uint32_t t) { return (t & 1u) | ((t >> 2) & 1u) << 1 | ((t >> 1) & 1u) << 2; }
constexpr uint32_t swap_xz(uint32_t t) { return (t & 2u) | ((t >> 2) & 1u) | (t & 1u) << 2; }

// One level: the key digit for octant o in state s, and the next state.
constexpr uint32_t step(const State& s, uint32_t o, State& next) {
    const uint32_t t = image(s.map, o);
    const uint32_t a = (t >> 2) & 1u, b = (t >> 1) & 1u, c = t & 1u;
    // Gray code of the level, then the fold of the parity above it
    const uint32_t gx = a, gy = a ^ b, gz = a ^ b ^ c;
    const uint32_t digit = ((gx ^ s.f) << 2) | ((gy ^ s.f) << 1) | (gz ^ s.f);
    next.f = s.f ^ gz;
    uint32_t map = 0;
    for (uint32_t k = 0; k < 8; ++k) {
        uint32_t v = image(s.map, k);
        if (a) v = flip_x(v);
        v = b ? flip_x(v) : swap_xy(v);
        v = c ? flip_x(v) : swap_xz(v);
        map |= v << (3 * k);
    }
    next.map = map;
    return digit;
}

constexpr int find_or_add(State* states, int& n, const State& s) {
    for (int k = 0; k < n; ++k)
        if (states[k].map == s.map && states[k].f == s.f) return k;
    states[n] = s;
    return n++;
}

}  // namespace hilbert_fsm

constexpr HilbertTables make_hilbert_tables() {
    using namespace hilbert_fsm;
    HilbertTables T{};
    State states[HT_MAX_STATES + 1] = {};
    uint32_t ident = 0;
    for (uint32_t k = 0; k < 8; ++k) ident |= k << (3 * k);
    int n = 0;
    find_or_add(states, n, State{ident, 0u});
    // one-level transitions; new states are appended and visited in turn
    for (int s = 0; s < n && n <= HT_MAX_STATES; ++s) {
        for (uint32_t o = 0; o < 8; ++o) {
            State nx{};
            const uint32_t d = step(states[s], o, nx);
            const int id = find_or_add(states, n, nx);
            if (id < HT_MAX_STATES) T.one[s * 8 + o] = (uint16_t)(d | (uint32_t)id << 6);
        }
    }
    T.nstates = n;
    for (int s = 0; s < n && s < HT_MAX_STATES; ++s) {
        for (uint32_t hi = 0; hi < 8; ++hi) {
            const uint32_t e1 = T.one[s * 8 + hi];
            const int s1 = (int)(e1 >> 6);
            for (uint32_t lo = 0; lo < 8; ++lo) {
                const uint32_t e2 = T.one[s1 * 8 + lo];
                T.two[s * 64 + (hi << 3 | lo)] = (uint16_t)(((e1 & 7u) << 3) | (e2 & 7u) | (e2 >> 6) << 6);
            }
        }
    }
    return T;
}

constexpr HilbertTables kHilbertTables = make_hilbert_tables();
static_assert(kHilbertTables.nstates <= HT_MAX_STATES, "the transform has at most 96 states");

}  // namespace tess
