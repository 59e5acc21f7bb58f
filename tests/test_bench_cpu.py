"""bench.py's algorithmic byte and flop counts (the roofline numerators),
checked against counts written out tensor by tensor for the Mamba-2
1.3B-shaped layer (batch 4 x 2048 tokens, 64 heads x P=64, N=128, one group,
chunk 256) and the batch-256 decode.  No GPU is used."""
import bench

b, L, H, P, N, G, Q = 4, 2048, 64, 64, 128, 1, 256
tok = b * L


def test_prefill_bytes_tensor_by_tensor():
    x = tok * H * P * 2                  # bf16
    y = tok * H * P * 4                  # fp32
    bc = 2 * tok * G * N * 2             # B and C, bf16
    dt_raw = tok * H * 2
    final = b * H * N * P * 4
    assert bench.prefill_bytes(b, L, H, P, N, G, 2, 4, 4) == x + y + bc + dt_raw + final == 214_958_080


def test_prefill_flops_per_chunk():
    nc = L // Q
    cb = G * 2 * Q * Q * N               # C B^T, once per group
    mx = H * 2 * Q * Q * P               # the masked matrix times X
    states = H * 4 * Q * N * P           # chunk state in and C h out
    assert bench.prefill_flops(b, L, H, P, N, G, Q) == b * nc * (cb + mx + states)


def test_backward_bytes_tensor_by_tensor():
    reads = tok * H * P * 2 * 2 + tok * H * 2 + 2 * tok * G * N * 2 + b * H * N * P * 4   # x, dy, dt_raw, B, C, dfinal
    writes = tok * H * P * 4 + tok * H * 4 + 2 * tok * G * N * 4                          # dx, ddt_raw, dB, dC (fp32)
    assert bench.backward_bytes(b, L, H, P, N, G, 2, 4, 4) == reads + writes == 292_552_704


def test_backward_flops_are_three_scans():
    # the adjoint scan has the forward's shape; the two transposed scans have
    # headdim N, dstate P and one group per head
    main = bench.prefill_flops(b, L, H, P, N, G, Q)
    transposed = bench.prefill_flops(b, L, H, N, P, H, Q)
    assert bench.backward_flops(b, L, H, P, N, G, Q) == main + 2 * transposed


def test_decode_bytes_state_read_and_write():
    bd, Hd, Pd, Nd, Gd = 256, 128, 64, 128, 8
    state = 2 * bd * Hd * Nd * Pd * 4
    io = bd * Hd * Pd * (2 + 4) + 2 * bd * Gd * Nd * 2 + bd * Hd * 2
    assert bench.decode_bytes(bd, Hd, Pd, Nd, Gd, 2, 4, 4) == state + io == 2_161_180_672


def test_executed_flops_block_by_block():
    # 128-token blocks; the head-pair kernel forms C B^T once per pair of heads, the
    # single-head kernel once per head; per head C h, the chunk state and M X each
    # run on the bf16 hi and lo parts of the operand computed in the kernel
    nblk = L // 128
    s = 2 * 128 * 128 * N
    per_head = 2 * (2 * 128 * N * P) + 2 * (2 * 128 * N * P) + 2 * (2 * 128 * 128 * P)
    assert bench.executed_flops(b, L, H, P, N, G, 2) == b * nblk * (H // 2 * s + H * per_head)
    assert bench.executed_flops(b, L, H, P, N, G, 0) == b * nblk * (H * s + H * per_head)


def test_backward_executed_flops_by_instruction():
    # per (b, h, 128-token block): M = 128 MMAs with K = 16 steps, 2*M*N*K flops each;
    # S^T (N 128, 8 steps), X dY^T (N 128, 4), B Ge and C h0 (N 64, 8, hi + lo each),
    # Mt dY (N 64, 8, hi + lo), dS^T C and dS B (N 128, 8, hi + lo each), the weighted
    # products (N 128, 4 steps, three per accumulator, two accumulators); per
    # direction one state update (N 64, 8 steps, hi + lo)
    nblk = L // 128
    f = lambda n, steps: steps * 2 * 128 * n * 16
    unit = f(128, 8) + f(128, 4) + 2 * 2 * f(64, 8) + 2 * f(64, 8) + 2 * 2 * f(128, 8) + 3 * 2 * f(128, 4)
    state = 2 * f(64, 8)
    assert bench.backward_executed_flops(b, L, H, P, N, G) == b * H * nblk * (unit + 2 * state)


def test_handoff_prefill_bytes():
    bb, LL, HH, GG = 512, 1024, 128, 8
    t = bb * LL
    x, y = t * HH * P * 2, t * HH * P * 4
    bc, dt_raw = 2 * t * GG * N * 2, t * HH * 2
    final = bb * HH * N * P * 2          # bf16 state handed to the decode steps
    assert bench.prefill_bytes(bb, LL, HH, P, N, GG, 2, 4, 2) == x + y + bc + dt_raw + final


def test_main_reads_no_name_bound_only_inside_the_layer_legs():
    """bench.main() nests the 1.3B-layer legs in a function (so that --layer-only
    can run them alone); a name bound only inside it is undefined outside, which
    only a full GPU run would otherwise reveal."""
    import ast
    tree = ast.parse(open(bench.__file__).read())
    main = next(n for n in tree.body if isinstance(n, ast.FunctionDef) and n.name == "main")
    inner = next(n for n in ast.walk(main) if isinstance(n, ast.FunctionDef) and n.name == "layer_legs")
    inner_ids = {id(n) for n in ast.walk(inner)}

    def bound(nodes):
        out = set()
        for n in nodes:
            if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Store):
                out.add(n.id)
            elif isinstance(n, ast.arg):
                out.add(n.arg)
            elif isinstance(n, (ast.FunctionDef, ast.Import, ast.ImportFrom)):
                out |= {n.name} if isinstance(n, ast.FunctionDef) else {a.asname or a.name for a in n.names}
        return out

    outer_nodes = [n for n in ast.walk(main) if id(n) not in inner_ids]
    only_inner = bound(n for stmt in inner.body for n in ast.walk(stmt)) - bound(outer_nodes) - {inner.name}
    read_outside = {n.id for n in outer_nodes if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Load)}
    assert not (only_inner & read_outside), sorted(only_inner & read_outside)
