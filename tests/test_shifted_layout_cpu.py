"""The shifted kernels' addressing, replayed on the host for the library's own plans.

Contiguous tensors off 16-byte boundaries run the 16-byte kernels in the
shifted layout: the packed layout laid over the output from position sh (the
output's offset in elements), each input read as one or two aligned 16-byte
chunks per output vector. This test replays, per thread of the plan that
dyt_plan_query returns, the rows it visits, the chunks it copies (plain copies
on its whole-vector rows, checked copies elsewhere), the output elements it
stores, the columns it assigns and the partial-sum slots it writes, with the
same arithmetic as the kernels (dyt_async.cuh, shifted kernels), and checks:
- every byte read lies inside its tensor;
- every output element is stored exactly once, at its own address;
- every stored element's input bytes were copied in the same row step;
- element e of the matrix gets column e mod N;
- its partial-sum slot is congruent to that column mod N (what the finalize
  relies on).
Host arithmetic only: no device is touched.
"""
import pytest

from tests.test_abi_cpu import _lib


def _cdiv(a, b):
    return -(-a // b)


def _chunk_width(B, RL, ncc, NV):
    # vector-columns per column chunk: equal chunks in whole warps
    return B if RL > 1 else min(B, _cdiv(_cdiv(NV, ncc), 32) * 32)


def replay(dyt, M, N, xd, hx, hd, ho, backward, sms=3):
    es = 4 if xd == 0 else 2
    vec = 16 // es
    p = dyt.dyt_plan_query(M, N, xd, 0, int(backward), 2, sms, 1, shift=ho)
    assert p["shifted"] == 1 and p["shift"] == ho
    B, RL, ncc, nrg, grid, pk = (p[k] for k in ("block", "row_lanes", "col_chunks", "row_groups", "grid", "pack_rows"))
    Np = pk * N                       # pitch of a row of the layout
    NV = Np // vec                    # 16-byte vectors per row of the layout
    sh, total = ho, M * N + ho        # the matrix occupies positions [sh, total) of the layout
    Mp = _cdiv(total, Np)
    gq, grem = Mp // nrg, Mp % nrg
    cw = _chunk_width(B, RL, ncc, NV)
    bases = {"x": 1 << 20, "dy": 2 << 20, "o": 3 << 20}  # 16-byte aligned regions, one per tensor
    lo = {"x": bases["x"] + hx * es, "dy": bases["dy"] + hd * es, "o": bases["o"] + ho * es}
    hi = {k: v + M * N * es for k, v in lo.items()}
    ins = ["x", "dy"] if backward else ["x"]
    frame = {}
    for k in ins:  # where position 0 of the layout falls in each input: aligned chunk base, byte offset d
        f = lo[k] - sh * es
        frame[k] = (f - (f & 15), f & 15)
    out_base = lo["o"] - sh * es
    assert out_base % 16 == 0
    stored = set()
    for blk in range(grid):
        for tid in range(B):
            rl, cvl, live = (tid // NV, tid % NV, tid // NV < RL) if RL > 1 else (0, tid, True)
            for item in range(blk, nrg * ncc, grid):
                cc, rg = (0, item) if ncc == 1 else (item % ncc, item // ncc)
                rb = rg * gq + min(rg, grem)
                re = rb + gq + (1 if rg < grem else 0)
                cv = cc * cw + cvl
                if not (live and cvl < cw and cv < NV):
                    continue
                c0 = cv * vec
                first = rb + rl
                n = 0 if first >= re else _cdiv(re - first, RL)
                assert n <= 2048
                if n > 0 and total - ((first + (n - 1) * RL) * Np + c0) <= 0:
                    n -= 1  # a last vector wholly past the matrix is not visited
                c = c0 - sh
                while c < 0:
                    c += N
                cols = [(c + e) % N for e in range(vec)]
                pos0, dpos, step = first * Np + c0, RL * Np, RL * Np * es

                def chunk(k, name):
                    return frame[name][0] + (first * Np + c0) * es + k * step

                def lo_ok(k):
                    return pos0 + k * dpos >= sh and all(chunk(k, m) >= lo[m] for m in ins)

                def hi_ok(k):
                    return pos0 + k * dpos + vec <= total and all(
                        chunk(k, m) + (32 if frame[m][1] else 16) <= hi[m] for m in ins)

                k_lo = 0
                while k_lo < n and not lo_ok(k_lo):
                    k_lo += 1
                k_hi = n
                while k_hi > k_lo and not hi_ok(k_hi - 1):
                    k_hi -= 1
                for k in range(n):
                    fast = k_lo <= k < k_hi
                    got = {}
                    for m in ins:
                        a, d = chunk(k, m), frame[m][1]
                        bytes_ = set()
                        for ca in ([a, a + 16] if d else [a]):
                            if fast:  # plain 16-byte copy
                                bytes_.update(range(ca, ca + 16))
                            elif ca >= hi[m] or ca + 16 <= lo[m]:
                                continue  # holds none of the tensor: not copied
                            elif ca >= lo[m]:  # the tensor ends here: its leading bytes, zero-filled slot
                                bytes_.update(range(ca, ca + min(16, hi[m] - ca)))
                            else:  # the tensor starts here: element by element from its first byte
                                assert (lo[m] - ca) % es == 0
                                bytes_.update(range(lo[m], min(hi[m], ca + 16)))
                        assert all(lo[m] <= b < hi[m] for b in bytes_), ("read outside", m)
                        got[m] = (a + d, bytes_)
                    pos = pos0 + k * dpos
                    for e in range(vec):
                        real = sh <= pos + e < total
                        if fast:
                            assert real
                        if not real:
                            continue  # masked: neither stored nor summed
                        f = pos + e - sh  # flat index in the matrix
                        assert out_base + (pos + e) * es == lo["o"] + f * es
                        assert f not in stored, "stored twice"
                        stored.add(f)
                        assert cols[e] == f % N
                        for m in ins:
                            start, bytes_ = got[m]
                            for b in range(start + e * es, start + (e + 1) * es):
                                assert b in bytes_, "an input byte was not copied"
                                assert (b - lo[m]) // es == f
                        q = c0 + e  # partial-sum slot of this position
                        slot = q - sh if q >= sh else q - sh + Np
                        assert slot % N == cols[e]
    assert len(stored) == M * N


CASES = [(M, N) for N in (1, 3, 8, 17, 32, 100, 255) for M in (1, 3, 9)] + [(33, 17), (5, 520), (3, 1031)]


@pytest.mark.parametrize("xd", [0, 1])
@pytest.mark.parametrize("M,N", CASES)
def test_shifted_addressing_stays_inside_every_tensor(xd, M, N):
    dyt = _lib()
    vec = 4 if xd == 0 else 8
    for backward in (False, True):
        for ho in range(vec):
            for hx in sorted({0, 1, vec - 1, ho}):
                for hd in (sorted({0, ho, vec - 1}) if backward else [0]):
                    replay(dyt, M, N, xd, hx, hd, ho, backward)


@pytest.mark.parametrize("M,N,xd", [(3, 4104, 1), (2, 4099, 1), (4, 2051, 0)])
def test_shifted_addressing_with_column_chunks(M, N, xd):
    # rows wider than a CTA's vectors: several column chunks per row
    dyt = _lib()
    vec = 4 if xd == 0 else 8
    for ho in (0, 1, vec - 1):
        for hx in (0, 1):
            for backward in (False, True):
                replay(dyt, M, N, xd, hx, hx, ho, backward, sms=5)


def _round_up(a, b):
    return _cdiv(a, b) * b


def replay_rowframe(dyt, M, N, xd, offs, lds, backward, sms=3):
    """The row frame: strided rows whose pitches are whole 16-byte vectors,
    each row laid out on its own from position sh (the output's offset) of a
    row of ceil((N + sh) / vec) vectors; with N a multiple of vec, sh > 0 and
    every input at the output's offset, of N / vec vectors, the first one also
    holding the row's last sh elements at its positions 0 .. sh - 1 (the
    wrapped vector-column). offs / lds: each tensor's offset past a 16-byte
    boundary and its pitch, in elements."""
    es = 4 if xd == 0 else 2
    vec = 16 // es
    ho = offs["o"]
    ins = ["x", "dy"] if backward else ["x"]
    layout = 3 if all(offs[m] == ho for m in ins) else 4
    p = dyt.dyt_plan_query(M, N, xd, 0, int(backward), layout, sms, 1, shift=ho)
    wrap = p["shifted"] == 3
    assert wrap == (layout == 3 and ho > 0 and N % vec == 0)
    if ho or N % vec:
        assert p["shifted"] in (2, 3) and p["shift"] == ho and p["pack_rows"] == 1
    B, RL, ncc, nrg, grid = (p[k] for k in ("block", "row_lanes", "col_chunks", "row_groups", "grid"))
    NV = N // vec if wrap else _cdiv(N + ho, vec)  # vectors of a row's frame
    assert ncc == (1 if RL > 1 else _cdiv(NV, B))
    gq, grem = M // nrg, M % nrg
    cw = _chunk_width(B, RL, ncc, NV)
    bases = {"x": 1 << 24, "dy": 2 << 24, "o": 3 << 24}
    lo = {k: bases[k] + offs[k] * es for k in bases}    # row 0 of each tensor
    for k in bases:
        assert lds[k] >= N and lds[k] * es % 16 == 0
    frame = {}
    for k in ins:  # where position 0 of row 0's frame falls: aligned chunk base, byte offset d
        f = lo[k] - ho * es
        frame[k] = (f - (f & 15), f & 15)
        if offs[k] == ho:
            assert frame[k][1] == 0  # same offset as the output: single chunks
    assert (lo["o"] - ho * es) % 16 == 0
    stored = set()
    for blk in range(grid):
        for tid in range(B):
            rl, cvl, live = (tid // NV, tid % NV, tid // NV < RL) if RL > 1 else (0, tid, True)
            for item in range(blk, nrg * ncc, grid):
                cc, rg = (0, item) if ncc == 1 else (item % ncc, item // ncc)
                rb = rg * gq + min(rg, grem)
                re = rb + gq + (1 if rg < grem else 0)
                cv = cc * cw + cvl
                if not (live and cvl < cw and cv < NV):
                    continue
                c0 = cv * vec
                first = rb + rl
                n = 0 if first >= re else _cdiv(re - first, RL)
                assert n <= 2048
                w = wrap and cv == 0
                if w:  # positions 0 .. ho - 1: the row's last ho columns
                    mask = [True] * vec
                    cols = [(c0 + e - ho) % N for e in range(vec)]
                else:
                    mask = [ho <= c0 + e < N + ho for e in range(vec)]
                    cols = [min(max(c0 + e - ho, 0), N - 1) for e in range(vec)]
                assert any(mask)
                # the tensors' spans, first element to last: the copies may read
                # the bytes between rows, never outside a span
                span = {m: (lo[m], lo[m] + ((M - 1) * lds[m] + N) * es) for m in ins}

                def chunk(k, m):
                    return frame[m][0] + c0 * es + (first + k * RL) * lds[m] * es

                def chunks(k, m):
                    a = chunk(k, m)
                    return [a] + ([a + 16] if frame[m][1] else []) + ([a + N * es] if w else [])

                def ok(k):
                    return all(chunks(k, m)[0] >= span[m][0] and chunks(k, m)[-1] + 16 <= span[m][1] for m in ins)

                k_lo = 0
                while k_lo < n and not ok(k_lo):
                    k_lo += 1
                k_hi = n
                while k_hi > k_lo and not ok(k_hi - 1):
                    k_hi -= 1
                assert k_lo <= 1 and k_hi >= n - 1  # only the tensors' first and last rows are checked
                for k in range(n):
                    row = first + k * RL
                    got = {}
                    for m in ins:
                        rlo = lo[m] + row * lds[m] * es
                        slo, shi = span[m]
                        a, d = chunk(k, m), frame[m][1]
                        assert a % 16 == 0
                        bytes_ = set()
                        for ca in chunks(k, m):
                            assert ca % 16 == 0
                            if k_lo <= k < k_hi:
                                bytes_.update(range(ca, ca + 16))
                            elif ca >= shi or ca + 16 <= slo:
                                continue
                            elif ca >= slo:
                                bytes_.update(range(ca, ca + min(16, shi - ca)))
                            else:
                                assert (slo - ca) % es == 0
                                bytes_.update(range(slo, min(shi, ca + 16)))
                        assert all(slo <= b < shi for b in bytes_), ("read outside the tensor", m)
                        got[m] = (a + d, rlo, bytes_)
                    out_row = lo["o"] + row * lds["o"] * es
                    out_frame = (lo["o"] - ho * es) + row * lds["o"] * es
                    for e in range(vec):
                        if not mask[e]:
                            continue  # the row's padding: neither stored nor summed
                        col = cols[e]
                        tail = w and e < ho  # stored N elements on, from the second chunk
                        assert out_frame + (c0 + e + (N if tail else 0)) * es == out_row + col * es
                        assert (row, col) not in stored, "stored twice"
                        stored.add((row, col))
                        if not w:
                            assert col == c0 + e - ho
                        for m in ins:
                            start, rlo, bytes_ = got[m]
                            src = start + (N * es if tail else 0) + e * es
                            for b in range(src, src + es):
                                assert b in bytes_, "an input byte was not copied"
                                assert (b - rlo) // es == col
                        # partial-sum slot: (position - sh) mod N, the column itself
                        assert (c0 + e - ho) % N == col
    assert len(stored) == M * N


RF_CASES = [(M, N) for N in (1, 3, 8, 17, 32, 100, 255) for M in (1, 3, 9)] + [(33, 17), (5, 520)]


@pytest.mark.parametrize("xd", [0, 1])
@pytest.mark.parametrize("M,N", RF_CASES)
def test_row_frame_addressing_stays_inside_every_row(xd, M, N):
    dyt = _lib()
    vec = 4 if xd == 0 else 8
    base = _round_up(N, vec)
    lds = {"x": base + vec, "dy": base, "o": base + 2 * vec}
    for backward in (False, True):
        for ho in range(vec):
            for hx in sorted({0, 1, vec - 1, ho}):
                for hd in (sorted({0, ho, vec - 1}) if backward else [0]):
                    replay_rowframe(dyt, M, N, xd, {"x": hx, "dy": hd, "o": ho}, lds, backward)


@pytest.mark.parametrize("M,N,xd", [(3, 4104, 1), (2, 4099, 1), (4, 2051, 0)])
def test_row_frame_addressing_with_column_chunks(M, N, xd):
    dyt = _lib()
    vec = 4 if xd == 0 else 8
    base = _round_up(N, vec)
    lds = {"x": base, "dy": base + vec, "o": base + vec}
    for ho in (0, 1, vec - 1):
        for hx in (0, 1):
            for backward in (False, True):
                replay_rowframe(dyt, M, N, xd, {"x": hx, "dy": hx, "o": ho}, lds, backward, sms=5)


def _period(ld, es):
    r = (ld * es) % 16
    return 1 if r == 0 else 16 // (r & -r)


@pytest.mark.parametrize("xd,N,lds,offs", [
    (1, 24, (26, 26, 26), (0, 0, 0)),     # 52 bytes: 4 phases
    (1, 40, (44, 44, 52), (1, 1, 1)),     # 88 / 104 bytes: 2 phases, every tensor one element off
    (1, 17, (19, 21, 23), (0, 3, 5)),     # odd pitches: 8 phases
    (0, 10, (10, 14, 18), (0, 1, 2)),     # fp32, x adjacent: 4 phases
    (0, 100, (102, 102, 106), (3, 3, 1)),  # 2 phases
])
def test_phase_plans_stay_inside_every_tensor(xd, N, lds, offs):
    # A strided call whose pitches are not whole 16-byte vectors runs rows j,
    # j + k, ... (k the longest pitch period) as k matrices of pitch k * ld.
    # Each phase is an ordinary strided call at its own offsets: replay the
    # library's plan for it and check that the phases cover every row once.
    dyt = _lib()
    es = 4 if xd == 0 else 2
    k = max(_period(ld, es) for ld in lds)
    assert k > 1
    M = 3 * k + 1
    ldx, ldd, ldo = lds
    covered = []
    for j in range(k):
        Mj = (M - j + k - 1) // k
        covered += [j + i * k for i in range(Mj)]
        # phase j starts j rows in: its offset past a 16-byte boundary, in elements
        sub_offs = {m: ((offs[i] + j * lds[i]) * es % 16) // es for i, m in enumerate(("x", "dy", "o"))}
        sub_lds = {"x": k * ldx, "dy": k * ldd, "o": k * ldo}
        for m in sub_lds:
            assert sub_lds[m] * es % 16 == 0  # every phase's pitch is a whole number of vectors
        for backward in (False, True):
            replay_rowframe(dyt, Mj, N, xd, sub_offs, sub_lds, backward)
    assert sorted(covered) == list(range(M))
