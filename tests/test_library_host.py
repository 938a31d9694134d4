"""Host-side checks of libe3conv.so (no GPU needed): exports, plans, CG tables,
path enumeration, code generation, error codes."""
import ctypes
import os
import re

import numpy as np
import pytest

import equivariant_graph_message_b200 as e3
import oracle
from workloads import ORDER, SPECS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "e3conv.h")).read()
    return sorted(set(re.findall(r"^E3CONV_API\s+[\w\s\*]*?\b(e3conv_\w+)\s*\(", text, re.M)))


def test_library_exports_every_declared_symbol():
    declared = _declared_symbols()
    assert len(declared) >= 20
    lib = ctypes.CDLL(e3.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(e3.EXPORTED) == declared
    assert e3.version() == 1


def test_strerror_covers_codes():
    for code in range(10):
        assert e3._strerror(code).decode() not in ("", "unknown error code")
    assert e3._strerror(99).decode() == "unknown error code"


@pytest.mark.parametrize("name", ORDER)
def test_paths_match_oracle(name):
    s = SPECS[name]
    c = e3.Conv(s.irreps_node, s.irreps_sh, s.irreps_out, 3.0)
    pl = oracle.plan(s.irreps_node, s.irreps_sh, s.irreps_out)
    assert (c.C, c.nx, c.ny, c.nout, c.num_paths) == (pl.C, pl.nx, pl.ny, pl.nout, len(pl.paths))
    assert c.num_paths == s.num_paths and c.nx == s.nx
    for q, r in zip(c.paths, pl.paths):
        assert (q.l1, q.p1, q.l2, q.l3, q.p3, q.x_off, q.out_off) == \
               (r.l1, r.p1, r.l2, r.l3, r.p3, r.x_off, r.out_off)
    assert c.outputs == [tuple(o) for o in pl.outputs]


@pytest.mark.parametrize("norm", ["SQRT_DIM_OUT", "NONE"])
def test_cg_tables_match_oracle_to_1e13(norm):
    # Racah closed form + real-basis map (library) vs intertwiner null space (oracle)
    irreps = ("1x0e+1x1o+1x2e+1x3o+1x4e+1x1e+1x2o", "1x0e+1x1o+1x2e+1x3o+1x4e",
              "+".join(f"1x{l}{p}" for l in range(7) for p in "eo"))
    c = e3.Conv(*irreps, 1.0, normalization=norm)
    assert c.num_paths > 60
    for p, q in enumerate(c.paths):
        np.testing.assert_allclose(c.cg(p), oracle.cg(q.l1, q.l2, q.l3, norm), atol=1e-13,
                                   err_msg=str(q))


def test_output_filter_drops_unreachable_irreps():
    c = e3.Conv("2x0e+2x1o+2x2e", "1x0e+1x1o+1x2e+1x3o", "2x0e+2x0o+2x1e+2x1o+2x2e+2x2o", 1.0)
    assert (0, -1) not in [(l, p) for l, p, _ in c.outputs]
    assert c.nout == 17


@pytest.mark.parametrize("args,code", [
    (("4x0e+5x1o", "1x0e", "4x0e"), 2),            # unequal multiplicities
    (("4x0e", "1x0e+1x2e", "4x0e"), 2),            # edge degrees not consecutive
    (("4x0e", "1x0e+1x1e", "4x0e"), 2),            # wrong edge parity
    (("4x0e", "2x0e", "4x0e"), 2),                 # edge multiplicity != 1
    (("4x0e", "1x0e", "4x0o"), 2),                 # no path reaches the filter
    (("4x0e", "1x0e", "4x0e+4x0e"), 2),            # duplicate output irrep
    (("4x0q", "1x0e", "4x0e"), 2),                 # malformed
    (("4x0e", "1x0e", "3x0e"), 2),                 # output multiplicity != C
    (("", "1x0e", "4x0e"), 2),
    (("1x7e", "1x0e", "1x7e"), 3),                 # degree above 6
])
def test_create_errors(args, code):
    with pytest.raises(e3.E3ConvError) as ei:
        e3.Conv(*args, 1.0)
    assert ei.value.code == code


def test_create_rejects_bad_scalars():
    for avg in (0.0, -1.0, float("nan"), float("inf")):
        with pytest.raises(e3.E3ConvError) as ei:
            e3.Conv("1x0e", "1x0e", "1x0e", avg)
        assert ei.value.code == 1
    with pytest.raises(KeyError):
        e3.Conv("1x0e", "1x0e", "1x0e", 1.0, normalization="COMPONENT")
    h = ctypes.c_void_p()
    assert e3._create(ctypes.byref(h), b"1x0e", b"1x0e", b"1x0e", 1.0, 7) == 3
    assert not h.value


def _emulate_phase1(c, src, Y, expect_entries):
    """Runs every generated phase-1 table (one per coop group) on the host and checks the A
    slots against the dense CG tables; returns the number of entries seen."""
    seen = 0
    for sfx, items in re.findall(r"// A layout(\S*) \(entry: path i k slot\):(.*)", src):
        m = re.search(r"// A rounds" + re.escape(sfx) + r" \(lanes (\d+), mode (\d)\):(.*)", src)
        rw, mode, terms = int(m.group(1)), int(m.group(2)), [int(v) for v in m.group(3).split()]
        encoded = mode >= 2          # apply-order layouts: the slot travels in the first index
        entries = [tuple(int(v) for v in it.split(":")) for it in items.split()]
        tab = re.search(r"e3_atab" + re.escape(sfx) + r"\[\] = \{(.*?)\};", src, re.S).group(1)
        cells = [(int(a), int(b)) for a, b in re.findall(r"\{(-?\d+), (\d+)\}", tab)]
        slots = {}
        base = 0
        for r, nterms in enumerate(terms):
            for lane in range(rw):
                q = r * rw + lane
                if q >= len(entries):
                    continue
                v, slot = 0.0, q
                for term in range(nterms):
                    cb, j = cells[base + term * rw + lane]
                    if encoded and term == 0:
                        slot, j = j >> 8, j & 255
                    v += np.frombuffer(np.int32(cb).tobytes(), np.float32)[0] * Y[j]
                slots[slot] = v
            base += nterms * rw
        assert base == len(cells)
        assert len(slots) == len(entries)                 # distinct slots, one per entry
        for p, i, k, slot in entries:
            W = c.cg(p)
            l2 = c.paths[p].l2
            expect = sum(W[i, j, k] * Y[l2 * l2 + j] for j in range(W.shape[1]))
            assert abs(slots[slot] - expect) < 1e-6 * (1 + abs(expect)), (sfx, p, i, k)
        seen += len(entries)
    assert seen == expect_entries
    return seen


@pytest.mark.parametrize("layout", [0, 1, 2, 3])
@pytest.mark.parametrize("name", ["large_f16", "large_f32", "mace"])
def test_a_layouts_form_every_entry_and_load_within_the_area(name, layout):
    # every A layout: the generated phase-1 tables form each entry in its own slot; the
    # apply-order float layout (3) reads 16-byte groups that start on a multiple of four slots
    s = SPECS[name]
    c = e3.Conv(s.irreps_node, s.irreps_sh, s.irreps_out, 40.0, dtype=s.dtype)
    c.set_a_layout(layout)
    src = c.kernel_source()
    assert f"a_layout={layout}" in src and c.kernel_info()["local_bytes"] == 0
    na = sum(int((np.abs(c.cg(p)) > 1e-12).any(axis=1).sum()) for p in range(c.num_paths))
    _emulate_phase1(c, src, np.random.default_rng(layout).normal(size=c.ny), expect_entries=na)
    if layout == 3:
        starts = [int(v) for v in re.findall(r"const float4 a4_\d+ = \*reinterpret_cast<const float4\*>\(Aw \+ (\d+)\)", src)]
        assert starts and all(v % 4 == 0 for v in starts)
        slots = [int(it.split(":")[3]) for it in
                 re.search(r"// A layout \(entry: path i k slot\):(.*)", src).group(1).split()]
        assert max(starts) + 4 <= (max(slots) + 4) // 4 * 4


def test_generated_kernel_unrolls_every_coefficient():
    s = SPECS["large_f16"]
    c = e3.Conv(s.irreps_node, s.irreps_sh, s.irreps_out, 40.0, dtype="f16")
    nnz = sum(int((np.abs(c.cg(p)) > 1e-12).sum()) for p in range(c.num_paths))
    assert nnz == 611
    # contraction-first (the float32 path): one table entry per nonzero
    # A_p[i,k] = sum_j CG_p[i,j,k] Y_j, each applied to every channel pair
    c.set_tensor_cores(0)
    info = c.kernel_info()
    assert info["contract_first"] == 1 and info["stages"] >= 2 and info["local_bytes"] == 0
    src = c.kernel_source()
    na = sum(int((np.abs(c.cg(p)) > 1e-12).any(axis=1).sum()) for p in range(c.num_paths))
    assert na == 541
    # emulate the generated phase-1 table on the host: the slot each lane writes must
    # hold sum_j CG[i,j,k] Y_j of the (path, i, k) the layout names
    Y = np.random.default_rng(1).normal(size=c.ny)
    _emulate_phase1(c, src, Y, expect_entries=na)
    groups = info["channels_per_lane"] // 2
    assert src.count("fma2(") + src.count("mul2(") >= na * groups
    # per-lane products (contract_first = 0): every CG nonzero for every channel
    c.set_contract_first(0)
    info = c.kernel_info()
    assert info["contract_first"] == 0
    src = c.kernel_source()
    V = info["channels_per_lane"]
    n_fma = src.count("fmaf(")
    n_mul = len(re.findall(r"= c\d+ \* x", src)) + len(re.findall(r"= s_\d \* x", src))
    assert n_fma + n_mul >= nnz * V
    assert "e3conv_fwd" in src and "row_ptr" in src and "atomicAdd" not in src
    assert info["local_bytes"] == 0


@pytest.mark.parametrize("V,block", [(1, 64), (2, 256), (4, 128)])
def test_launch_config_recompiles(V, block):
    s = SPECS["mace"]
    c = e3.Conv(s.irreps_node, s.irreps_sh, s.irreps_out, 30.0)
    c.set_launch_config(V, block)
    info = c.kernel_info()
    assert info["channels_per_lane"] == V and info["block_threads"] == block
    with pytest.raises(e3.E3ConvError):
        c.set_launch_config(3, 0)
    with pytest.raises(e3.E3ConvError):
        c.set_launch_config(0, 100)


def test_host_only_plan_forward_reports_no_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present; covered by the GPU tests")
    c = e3.Conv("1x0e", "1x0e", "1x0e", 1.0)
    rc = e3._forward(c._h, ctypes.c_void_p(16), None, None, None, ctypes.c_void_p(16), 1,
                     ctypes.c_void_p(16), None)
    assert rc == 7
    ws = ctypes.c_size_t()
    assert e3._csr_ws(10, 5, ctypes.byref(ws)) == 0 and ws.value > 0


def test_forward_signature_has_no_host_edge_count():
    # e3conv_forward(plan, x, Y, s, senders, row_ptr, num_nodes, out, stream): the edge count
    # is row_ptr[num_nodes], read on the device only
    import inspect
    header = open(os.path.join(ROOT, "include", "e3conv.h")).read()
    decl = header[header.index("E3CONV_API int e3conv_forward("):]
    decl = decl[:decl.index(";")]
    args = [a.split()[-1].strip("*") for a in decl[decl.index("(") + 1:decl.rindex(")")].split(",")]
    assert args == ["plan", "node_features", "edge_sh", "edge_scalars", "senders",
                    "receiver_row_ptr", "num_nodes", "out", "stream"]
    assert len(e3._forward.argtypes) == 9
    assert "num_edges" not in inspect.signature(e3.Conv.forward_raw).parameters


def test_forward_argument_validation_precedes_device():
    c = e3.Conv("1x0e", "1x0e", "1x0e", 1.0)
    assert e3._forward(c._h, None, None, None, None, None, -1, None, None) == 1
    assert e3._forward(c._h, None, None, None, None, None, 0, None, None) == 0   # nothing to do
    assert e3._forward(c._h, None, None, None, None, None, 3, None, None) == 1
    # misaligned feature buffers
    assert e3._forward(c._h, ctypes.c_void_p(18), None, None, None, ctypes.c_void_p(16), 3,
                       ctypes.c_void_p(16), None) == 1
    assert e3._forward(c._h, ctypes.c_void_p(16), ctypes.c_void_p(20), None, None,
                       ctypes.c_void_p(16), 3, ctypes.c_void_p(16), None) == 1
    assert e3._build_csr(None, -1, 3, None, None, None, 0, None) == 1


def test_forward_rows_range_validation():
    c = e3.Conv("1x0e", "1x0e", "1x0e", 1.0)
    p16 = ctypes.c_void_p(16)
    fr = e3._forward_rows
    assert fr(c._h, p16, 10, p16, p16, p16, p16, -1, 5, p16, None) == 1      # begin < 0
    assert fr(c._h, p16, 10, p16, p16, p16, p16, 6, 5, p16, None) == 1       # end < begin
    assert fr(c._h, p16, 10, p16, p16, p16, p16, 0, 1 << 31, p16, None) == 1  # end >= 2^31
    assert fr(c._h, None, 10, None, None, None, None, 4, 4, None, None) == 0  # empty range
    assert fr(c._h, p16, 1 << 31, p16, p16, p16, p16, 0, 1, p16, None) == 1


def test_size_limits_rejected_on_host():
    # indices are int32: sizes of 2^31 and above are refused before any launch
    c = e3.Conv("1x0e", "1x0e", "1x0e", 1.0)
    p16 = ctypes.c_void_p(16)
    assert e3._forward(c._h, p16, p16, p16, p16, p16, 1 << 31, p16, None) == 1
    n = ctypes.c_size_t()
    assert e3._csr_ws(1 << 31, 10, ctypes.byref(n)) == 1
    assert e3._csr_ws(10, (1 << 31) - 1, ctypes.byref(n)) == 1
    assert e3._csr_ws((1 << 31) - 1, (1 << 31) - 2, ctypes.byref(n)) == 0
    cnt = ctypes.c_int()
    assert e3._csr_count((1 << 31) - 1, 100000, ctypes.byref(cnt)) == 0 and cnt.value > 0


def test_tensor_core_tables_emulated_on_host():
    # The tensor-core kernel writes A_p[i,k] = sum_j CG_p[i,j,k] Y_j into a
    # K-major B tile (K = node component, N = path output column); decode the
    # generated table and offsets and compare with the direct contraction.
    s = SPECS["large_f16"]
    c = e3.Conv(s.irreps_node, s.irreps_sh, s.irreps_out, 40.0, dtype="f16")
    c.set_tensor_cores(1)
    info = c.kernel_info()
    assert info["tensor_cores"] == 1 and info["local_bytes"] == 0
    src = c.kernel_source()
    ncols = int(re.search(r"ncols=(\d+)", src).group(1))
    tab = re.search(r"e3_btab\[\] = \{(.*?)\};", src, re.S).group(1)
    pairs = [(int(a), int(b)) for a, b in re.findall(r"\{(-?\d+), (\d+)\}", tab)]
    offs = [int(v) for v in re.search(r"e3_boff\[\] = \{(.*?)\};", src, re.S).group(1)
            .replace("\n", "").split(",") if v.strip()]
    Y = np.random.default_rng(3).normal(size=c.ny)
    B = np.zeros((16, ncols))
    lanes = int(re.search(r"producer_threads=(\d+)", src).group(1))
    loads = re.findall(r"const int2 k(\d+)_(\d+) = __ldg\(&e3_btab\[(\d+) \+ tl\]\);", src)
    nrounds = max(int(r) for r, _, _ in loads) + 1
    assert nrounds == -(-541 // lanes)
    for r in range(nrounds):
        bases = [int(b) for rr, _, b in loads if int(rr) == r]
        for lane in range(lanes):
            off = offs[r * lanes + lane]
            if off < 0:
                continue
            v = sum(np.frombuffer(np.int32(pairs[b + lane][0]).tobytes(), np.float32)[0] *
                    Y[pairs[b + lane][1]] for b in bases)
            n = (off // 256) * 8 + (off % 128) // 16           # K-major core-matrix layout
            i = ((off % 256) // 128) * 8 + (off % 16) // 2
            assert B[i, n] == 0
            B[i, n] = v
    order = list(range(len(c.paths)))                # T columns in path order
    expect = np.zeros((16, ncols))
    col = 0
    for p in order:
        q = c.paths[p]
        W = c.cg(p)
        d1, d2, d3 = W.shape
        for i in range(d1):
            for k in range(d3):
                expect[q.x_off + i, col + k] = W[i, :, k] @ Y[q.l2 ** 2:q.l2 ** 2 + d2]
        col += d3
    np.testing.assert_allclose(B, expect, atol=1e-5)
    assert (np.abs(expect) > 1e-9).sum() == 541


def test_binding_rejects_host_tensors_before_any_library_call():
    # host pointers never reach a kernel: every tensor is checked (CUDA, device, dtype,
    # contiguity, size) in the binding
    import torch
    c = e3.Conv("4x0e+4x1o", "1x0e+1x1o+1x2e", "4x0e+4x1o", 5.0)
    N, E = 3, 4
    x = torch.zeros(N, c.nx, c.C)
    Y = torch.zeros(E, c.ny)
    s = torch.zeros(E, c.num_paths, c.C)
    snd = torch.zeros(E, dtype=torch.int32)
    rp = torch.zeros(N + 1, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        c.forward(x, Y, s, snd, rp)
    with pytest.raises(ValueError, match="CUDA tensor"):
        e3.build_csr(torch.zeros(E, dtype=torch.int32), N)
    with pytest.raises(ValueError, match="CUDA tensor"):
        e3.build_csr_noalloc(torch.zeros(E, dtype=torch.int32), N)
    with pytest.raises(ValueError, match="CUDA tensor"):
        e3.permute_rows(torch.zeros(E, 2), torch.zeros(E, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA tensor"):
        e3.csr_check(torch.zeros(16, dtype=torch.uint8))


def test_tensor_core_kernels_fit_for_eligible_irreps_sets():
    # float16, C = 128 sets of up to four node irreps (nx <= 16) with Y l <= 3: the
    # tensor-core kernel compiles without spills, its teams' T columns fit the 512 of tensor
    # memory, its ring stages start on 1024-byte boundaries (128-byte swizzle) and the block
    # fits the 227 KB of shared memory
    import itertools
    irs = ["0e", "1o", "2e", "3o", "0o", "1e", "2o", "3e"]
    out_all = "+".join("128x" + r for r in irs)
    sh3 = "1x0e+1x1o+1x2e+1x3o"
    eligible = [combo for k in (1, 2, 3, 4) for combo in itertools.combinations(irs, k)
                if sum(2 * int(r[0]) + 1 for r in combo) <= 16]
    assert len(eligible) == 130
    # a deterministic subset (each compile takes seconds): every 12th set, the two sets that
    # need the two-team fallback and the benchmark's irreps
    picked = eligible[::12] + [("2e", "1e", "2o"), ("2e", "1e", "3e"), ("0e", "1o", "2e", "3o")]
    seen = 0
    for combo in picked:
        c = e3.Conv("+".join("128x" + r for r in combo), sh3, out_all, 10.0, dtype="f16")
        c.set_tensor_cores(1)
        info = c.kernel_info()
        assert info["tensor_cores"] == 1, combo
        assert info["local_bytes"] == 0, (combo, info)
        m = re.search(r"ncols=(\d+) teams=(\d+) tstride=(\d+) stages=(\d+) stage_bytes=(\d+) "
                      r"team_bytes=(\d+)", c.kernel_source())
        ncols, teams, tstride, stages, stage_bytes, team_bytes = map(int, m.groups())
        assert ncols % 16 == 0 and ncols <= 256 and tstride >= ncols and tstride % 32 == 0
        assert teams * tstride <= 512 and info["block_threads"] == 128 * teams
        assert stages >= 3 and stage_bytes % 1024 == 0 and team_bytes % 1024 == 0
        assert teams * team_bytes + 16 <= 227 * 1024
        seen += 1
    assert seen == len(picked)


@pytest.mark.parametrize("stages", [2, 4])
@pytest.mark.parametrize("combo", [("2e", "1e", "2o"), ("2e", "1e", "3e")])
def test_tensor_core_fallback_ladder_with_ring_depth(combo, stages):
    # With a requested ring depth (and the automatic block size that follows it) the kernel
    # is either the tensor-core kernel with no local memory, or the float32 staged kernel
    # with no local memory: never a tensor-core kernel that spills.  kernel_info describes the
    # source that was compiled, and its local bytes are the compiled stack frame.
    irs = ["0e", "1o", "2e", "3o", "0o", "1e", "2o", "3e"]
    c = e3.Conv("+".join("128x" + r for r in combo), "1x0e+1x1o+1x2e+1x3o",
                "+".join("128x" + r for r in irs), 10.0, dtype="f16")
    c.set_tensor_cores(1)
    c.set_launch_config(0, 0, stages)
    info = c.kernel_info()
    src = c.kernel_source()
    assert info["local_bytes"] == 0, info
    assert ("(tensor cores, teams)" in src) == bool(info["tensor_cores"])
    if info["tensor_cores"]:
        assert "tcgen05.mma" in src
    else:
        assert "(staged ring)" in src and "tcgen05" not in src


@pytest.mark.parametrize("lmax", [0, 1, 2, 3, 6])
def test_kernel_harmonics_match_the_oracle(lmax):
    # the polynomials the kernels evaluate from edge vectors (Bonnet recursion, exact
    # expansion in C++) against the oracle's Rodrigues-formula harmonics
    sh = "+".join(f"1x{l}{'eo'[l % 2]}" for l in range(lmax + 1))
    c = e3.Conv("4x0e", sh, "4x0e", 1.0)
    rng = np.random.default_rng(lmax)
    v = rng.normal(size=(40, 3)) * rng.uniform(0.01, 100, size=(40, 1))
    got = np.array([c.spherical_harmonics(q) for q in v])
    ref = oracle.sh(lmax, v / np.linalg.norm(v, axis=1, keepdims=True))
    np.testing.assert_allclose(got, ref, atol=1e-12)
    z = c.spherical_harmonics([0.0, 0.0, 0.0])
    assert z[0] == 1.0 and np.all(z[1:] == 0)


@pytest.mark.parametrize("name", ORDER)
def test_edge_vector_kernels_compile_for_every_workload(name):
    s = SPECS[name]
    c = e3.Conv(s.irreps_node, s.irreps_sh, s.irreps_out, 10.0, dtype=s.dtype)
    c.set_edge_vectors(1)
    assert c.edge_vectors
    info = c.kernel_info()
    assert info["local_bytes"] == 0
    src = c.kernel_source()
    assert "sqrtf(r2_)" in src and "const float* __restrict__ Y" in src


@pytest.mark.parametrize("dtype", ["f32", "f16"])
@pytest.mark.parametrize("lmax", [0, 1, 2, 3, 4])
def test_standalone_harmonics_kernel_compiles(lmax, dtype):
    # e3conv_edge_harmonics generates and compiles its kernel before it needs a device: on a
    # host it gets as far as "no device" (a compile failure would be E3CONV_ERR_COMPILE)
    sh = "+".join(f"1x{l}{'eo'[l % 2]}" for l in range(lmax + 1))
    c = e3.Conv("4x0e", sh, "4x0e", 1.0, dtype=dtype)
    rc = e3._edge_sh(c._h, ctypes.c_void_p(256), 5, ctypes.c_void_p(512), None)
    assert rc == 7, e3._last_error()                                      # E3CONV_ERR_NO_DEVICE
    assert e3._edge_sh(c._h, ctypes.c_void_p(256), 0, None, None) == 0    # empty: nothing to do
    assert e3._edge_sh(c._h, ctypes.c_void_p(258), 5, ctypes.c_void_p(512), None) == \
        1                                                                  # E3CONV_ERR_INVALID_ARG


@pytest.mark.parametrize("split", [2, 3, 4])
def test_path_split_tables_cover_every_entry_once(split):
    # the warps of a path-split team own disjoint output irreps; their tables together form
    # every A entry exactly once, each with the right value
    s = SPECS["large_f16"]
    c = e3.Conv(s.irreps_node, s.irreps_sh, s.irreps_out, 40.0, dtype="f16")
    c.set_path_split(split)
    src = c.kernel_source()
    assert f"path_split={split}" in src and c.kernel_info()["local_bytes"] == 0
    Y = np.random.default_rng(split).normal(size=c.ny)
    _emulate_phase1(c, src, Y, expect_entries=541)
    owned = [set(int(p) for p in re.findall(r"(\d+):\d+:\d+:\d+", items))
             for _, items in re.findall(r"// A layout(\S*) \(entry: path i k slot\):(.*)", src)]
    assert len(owned) == split
    assert set().union(*owned) == set(range(c.num_paths))
    assert sum(len(o) for o in owned) == c.num_paths          # each path in one warp


def test_linear_layer_host_validation():
    with pytest.raises(e3.E3ConvError):
        e3.IrrepsLinear("48x0e", "64x0e")                 # mul_in not 32, 64 or 128
    with pytest.raises(e3.E3ConvError):
        e3.IrrepsLinear("64x0e", "20x0e")                 # mul_out not a multiple of 16
    with pytest.raises(e3.E3ConvError):
        e3.IrrepsLinear("64x0e+64x0e", "64x0e")           # not regrouped
    with pytest.raises(e3.E3ConvError):
        e3.IrrepsLinear("64x0e+32x1o", "64x0e")           # unequal input multiplicities
    lin = e3.IrrepsLinear("64x0e+64x1o+64x2e", "32x2e+32x3o+32x0e")
    assert (lin.dim_in, lin.dim_out, lin.num_weight_blocks) == (64 * 9, 32 * 13, 2)
    with pytest.raises(ValueError):
        lin.set_weights([np.zeros((64, 32))])            # two matched irreps need two blocks


@pytest.mark.parametrize("ins,outs,fits", [
    ("128x0e+128x1o+128x2e+128x3o", "128x0e+128x1o+128x2e+128x3o", True),   # two stages
    ("64x0e+64x1o", "64x0e+64x1o", True),
    ("32x0e", "256x0e", True),
    ("64x0e", "64x0e+64x1o+64x1e", True),                     # unmatched outputs: zero tiles
    ("128x0e", "16x0e", False),                               # mul_out not a multiple of 32
    ("128x0e", "48x0e", False),
    ("128x0e+128x1o", "256x0e+256x1o", False),                # weights leave one stage
    ("64x0e", "+".join(f"64x{l}{'eo'[l % 2]}" for l in range(9)), False),  # 9 output irreps
])
def test_linear_kernel_choice(ins, outs, fits):
    # the tensor-map kernel takes a shape when mul_out is a multiple of 32 (32-column output
    # boxes), there are at most 8 output irreps (two tensor maps each as kernel parameters)
    # and two input stages fit in shared memory next to the weights and the staging tiles;
    # set_tma(False) always selects the row-per-thread kernel
    lin = e3.IrrepsLinear(ins, outs)
    assert lin.uses_tma == fits
    lin.set_tma(False)
    assert not lin.uses_tma
    lin.set_tma(True)
    assert lin.uses_tma == fits


@pytest.mark.parametrize("name", ORDER)
def test_backward_kernels_generate_for_every_workload(name):
    s = SPECS[name]
    c = e3.Conv(s.irreps_node, s.irreps_sh, s.irreps_out, 10.0, dtype=s.dtype)
    edges, nodes = c.backward_source(0), c.backward_source(1)
    parts = int(re.search(r"// part 0 of (\d+)", edges).group(1)) if "// part 0 of" in edges else 1
    for p in range(1, parts):          # kernels split over the output irreps: every launch
        later = c.backward_source(2 * p)
        assert f"// part {p} of {parts}" in later and "gY[le * " in later
        edges += later
        if "cp.async" in nodes:
            nodes += c.backward_source(2 * p + 1)
    with pytest.raises(e3.E3ConvError):
        c.backward_source(2 * parts)
    assert "e3conv_bwd_edges" in edges and "e3conv_bwd_nodes" in nodes
    # every CG nonzero appears once per channel of a lane in each kernel
    m = re.search(r"V=(\d+) TL=(\d+)", edges)
    V = int(m.group(1))
    nnz = sum(int((np.abs(c.cg(p)) > 1e-12).sum()) for p in range(c.num_paths))
    def a_terms(src):   # harmonic terms over all A_ik = sum_j c Y_j expressions
        return sum(len(re.findall(r"\by\d+\b", m))
                   for m in re.findall(r"const unsigned long long A_ = bc\((.*)\);", src))
    if "cp.async" in nodes:
        # staged nodes kernel: each nonzero appears once in its A_ik (applied to u_k = s g_k)
        assert a_terms(nodes) == nnz
    else:
        assert nodes.count(" = fmaf(") >= nnz * V
    if "cp.async" in edges:
        # staged edges kernel: each nonzero appears once in its A_ik = sum_j c Y_j and once in
        # dY_j += c W_ik (W already summed over the lane's channels)
        assert edges.count(", W_, dy") == nnz
        assert a_terms(edges) == nnz
    else:
        assert edges.count("dy") >= nnz * V


def test_backward_rejects_edge_vector_plans_and_wide_channels():
    c = e3.Conv("8x0e+8x1o", "1x0e+1x1o", "8x0e+8x1o", 1.0)
    c.set_edge_vectors(1)
    with pytest.raises(e3.E3ConvError):
        c.backward_source(0)
    wide = e3.Conv("256x0e", "1x0e+1x1o", "256x0e+256x1o", 1.0)   # float32, C > 128
    with pytest.raises(e3.E3ConvError):
        wide.backward_source(0)


def test_kernel_log_records_the_launch_shape_search():
    # e3conv_kernel_log: one line per compile of the search, then the kept compile's log
    s = SPECS["large_f16"]
    c = e3.Conv(s.irreps_node, s.irreps_sh, s.irreps_out, 40.0, dtype=s.dtype)
    log = c.kernel_log()
    lines = [ln for ln in log.splitlines() if ln.startswith("compile: ")]
    assert lines and all(re.search(r"block=\d+ V=\d+ team=\d+ stages=\d+ tc=\d regs=-?\d+ local=\d+", ln)
                         for ln in lines)
    info = c.kernel_info()
    assert f"block={info['block_threads']}" in lines[-1]
