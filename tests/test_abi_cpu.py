"""The C ABI without a GPU: the library loads, exports every declared symbol,
and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import sparse_kv_b200 as skv
from sparse_kv_b200 import DecodeArgs, _Art, _Window, _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x7F0000001000  # aligned, never dereferenced: every case fails validation first


def declared_functions():
    src = open(os.path.join(ROOT, "include", "sparsekv.h")).read()
    return re.findall(r"SKV_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["attn_decode", "attn_decode_static_ws", "attn_select_centroids", "attn_select_centroids2",
              "attn_merge_lse", "attn_route_layers", "skv_decode_workspace_size", "skv_decode_launches",
              "skv_decode_plan_info", "skv_strerror"]:
        assert n in names


def test_header_is_plain_c_and_cxx(tmp_path):
    # the boundary is a C ABI: the header compiles as C99 and as C++, and a C
    # program can name every entry point
    import shutil
    import subprocess
    src = tmp_path / "use.c"
    names = declared_functions()
    src.write_text('#include "sparsekv.h"\n' + "void* table[] = {" +
                   ", ".join(f"(void*){n}" for n in names) + "};\nint main(void) { return 0; }\n")
    inc = os.path.join(ROOT, "include")
    for cc, std in (("gcc", "-std=c99"), ("g++", "-std=c++17")):
        if shutil.which(cc) is None:
            pytest.skip(f"{cc} not found")
        args = [cc, std, "-Wall", "-Werror", "-fsyntax-only", "-I", inc]
        if cc == "g++":
            args += ["-x", "c++"]
        r = subprocess.run(args + [str(src)], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_binding_struct_matches_the_header(tmp_path):
    # the ctypes mirror of skv_decode_args has the C layout: same size and the
    # same offset for every field (checked with the C compiler's own offsetof)
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not found")
    fields = [f[0] for f in DecodeArgs._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "sparsekv.h"\nint main(void) {\n'
                   '  printf("size %zu\\n", sizeof(skv_decode_args));\n' +
                   "".join(f'  printf("{n} %zu\\n", offsetof(skv_decode_args, {n}));\n' for n in fields) +
                   "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                       check=True).stdout.splitlines())
    assert int(got["size"]) == ctypes.sizeof(DecodeArgs)
    for n in fields:
        assert int(got[n]) == getattr(DecodeArgs, n).offset, n
    # and the plan struct
    pf = [f[0] for f in skv.DecodePlan._fields_]
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "sparsekv.h"\nint main(void) {\n'
                   '  printf("size %zu\\n", sizeof(skv_decode_plan));\n' +
                   "".join(f'  printf("{n} %zu\\n", offsetof(skv_decode_plan, {n}));\n' for n in pf) +
                   "  return 0;\n}\n")
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                       check=True).stdout.splitlines())
    assert int(got["size"]) == ctypes.sizeof(skv.DecodePlan)
    for n in pf:
        assert int(got[n]) == getattr(skv.DecodePlan, n).offset, n


def test_library_exports_every_declared_symbol():
    L = skv.lib()
    for n in declared_functions():
        assert hasattr(L, n), n
    out = os.popen(f"nm -D --defined-only {_build.SO}").read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert set(declared_functions()) <= exported
    # nothing else leaks: only the declared C symbols are exported as functions
    assert not [s for s in exported if s.startswith("_Z")]


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(_build, "SO", "/nonexistent/libsparsekv.so")
    monkeypatch.setattr(skv, "_LIB", None)
    with pytest.raises(RuntimeError, match="libsparsekv.so not found"):
        skv.lib()


def good_args(**kw):
    a = DecodeArgs()
    a.q = a.k_pool = a.v_pool = a.block_table = a.seq_lens = a.out = a.lse = FAKE
    a.batch, a.q_tokens, a.q_heads, a.kv_heads, a.head_dim, a.block_size = 16, 1, 32, 8, 128, 64
    a.max_blocks, a.num_pages, a.max_seq_len = 512, 8192, 32768
    a.scale = 0.088
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def status(a):
    # a workspace-free configuration fails in validation; others fail at the workspace check
    return skv.lib().attn_decode(ctypes.byref(a), None)


@pytest.mark.parametrize("kw,want", [
    (dict(q=None), skv.SKV_EINVAL),
    (dict(out=None), skv.SKV_EINVAL),
    (dict(seq_lens=None), skv.SKV_EINVAL),
    (dict(batch=0), skv.SKV_EINVAL),
    (dict(q_heads=30), skv.SKV_EINVAL),
    (dict(q_heads=24), skv.SKV_EUNSUPPORTED),      # GQA group of 3
    (dict(head_dim=64), skv.SKV_EUNSUPPORTED),
    (dict(block_size=32), skv.SKV_EUNSUPPORTED),
    (dict(q_tokens=2, art=_Art(1, 1e-3, 1e-4, 4)), skv.SKV_EUNSUPPORTED),  # chunk + ART
    (dict(q_tokens=2, window=_Window(64, 4096)), skv.SKV_EUNSUPPORTED),   # chunk + window
    (dict(kv_shards=-1), skv.SKV_EINVAL),
    (dict(kv_shards=4), skv.SKV_EUNSUPPORTED),                            # shards need a chunk
    (dict(q=FAKE + 8), skv.SKV_EINVAL),            # misaligned
    (dict(k_pool=FAKE + 4), skv.SKV_EINVAL),
    (dict(max_blocks=100), skv.SKV_EINVAL),        # table narrower than max_seq_len
    (dict(scale=float("nan")), skv.SKV_EINVAL),
    (dict(art=_Art(1, -1.0, 1e-4, 4)), skv.SKV_EINVAL),
    (dict(art=_Art(1, float("nan"), 1e-4, 4)), skv.SKV_EINVAL),
    (dict(art=_Art(1, 1e-3, 1e-4, 0)), skv.SKV_EINVAL),
    (dict(art=_Art(1, 1e-3, 1e-4, 4), window=_Window(64, 4096)), skv.SKV_EUNSUPPORTED),
    (dict(order=FAKE, order_len=4, window=_Window(64, 4096)), skv.SKV_EUNSUPPORTED),
    (dict(seg_start=FAKE, n_seg=3), skv.SKV_EINVAL),  # seg_end missing
    (dict(window=_Window(-1, 4096)), skv.SKV_EINVAL),
    (dict(kv_begin=10, kv_end=5), skv.SKV_EINVAL),
    (dict(), skv.SKV_EWORKSPACE),                  # needs split-KV workspace, none given
])
def test_decode_rejects_on_host(kw, want):
    assert status(good_args(**kw)) == want


def test_workspace_size_query():
    L = skv.lib()
    full = good_args()
    n = L.skv_decode_workspace_size(ctypes.byref(full))
    # header (batch prefix) + per-warp partial records of 132 floats per head
    assert n > 0 and (n % 256) == 0 and n >= 16 * 8 * 16 * 4 * 132 * 4
    # ART: per (chunk, KV group): a look-back record of 12 floats and a partial
    # record of 132 floats per head, zeroed control words, and a scratch area of
    # at most 192 KB per resident CTA (2 per SM).  This shape (128 groups of 512
    # blocks, 296 CTAs: about 2.3 chunks of a group in flight) takes 16-block
    # chunks, since 32-block ones would read 74 blocks past a stop, over 1/12
    # of the walk.
    art = good_args(art=_Art(1, 1e-3, 1e-4, 4))
    items = 16 * 8 * (512 // 16)
    na = L.skv_decode_workspace_size(ctypes.byref(art))
    assert na >= items * 4 * (132 + 12) * 4 + (4 + 16 * 8 * (1 + 512 // 16 + 8)) * 4
    assert na < items * 4 * (132 + 12) * 4 + 64 * 1024 + 2 * 148 * 192 * 1024
    assert status(good_args(art=_Art(1, 1e-3, 1e-4, 4))) == skv.SKV_EWORKSPACE
    assert L.skv_decode_workspace_size(ctypes.byref(good_args(head_dim=64))) == 0
    small = good_args(workspace=FAKE, workspace_bytes=n - 16)
    assert status(small) == skv.SKV_EWORKSPACE


def test_decode_launch_count():
    # one kernel where the walk merges its own partials (small walks and
    # segment lists take the split schedule; a query chunk writes its results
    # directly), two where a record merge follows (large walks, ART)
    L = skv.lib()
    n = lambda a: L.skv_decode_launches(ctypes.byref(a))
    assert n(good_args()) == 2                                    # 128 groups x 512 tiles
    assert n(good_args(art=_Art(1, 1e-3, 1e-4, 4))) == 2
    small = good_args(batch=1, q_heads=8, kv_heads=2, max_seq_len=4096, max_blocks=64)
    assert n(small) == 1                                          # 2 groups x 64 tiles
    # the split schedule merges its pieces in the cluster's shared memory: no workspace
    assert L.skv_decode_workspace_size(ctypes.byref(small)) == 0
    assert n(good_args(seg_start=FAKE, seg_end=FAKE, n_seg=102)) == 1
    assert n(good_args(q_tokens=128)) == 1
    assert n(good_args(head_dim=64)) == 0


def test_select_and_merge_reject_on_host():
    L = skv.lib()
    sel = L.attn_select_centroids
    assert sel(FAKE, FAKE, FAKE, 8, 32, 8, 128, 1024, 2000, FAKE, FAKE, FAKE, None) == skv.SKV_EINVAL
    assert sel(FAKE, FAKE, FAKE, 8, 32, 8, 128, 8192, 102, FAKE, FAKE, FAKE, None) == skv.SKV_EUNSUPPORTED
    assert sel(FAKE, FAKE, FAKE, 8, 32, 8, 64, 1024, 102, FAKE, FAKE, FAKE, None) == skv.SKV_EUNSUPPORTED
    assert sel(None, FAKE, FAKE, 8, 32, 8, 128, 1024, 102, FAKE, FAKE, FAKE, None) == skv.SKV_EINVAL
    mer = L.attn_merge_lse
    assert mer(FAKE, FAKE, 0, 10, 128, FAKE, FAKE, None) == skv.SKV_EINVAL
    assert mer(FAKE, FAKE, 2, 10, 6, FAKE, FAKE, None) == skv.SKV_EINVAL
    assert mer(FAKE + 4, FAKE, 2, 10, 128, FAKE, FAKE, None) == skv.SKV_EINVAL
    assert mer(None, FAKE, 2, 10, 128, FAKE, FAKE, None) == skv.SKV_EINVAL


def test_route_rejects_on_host():
    L = skv.lib()
    r = L.attn_route_layers
    ok = (FAKE, FAKE, None, 32, 8, 128, 32, 128, 64, 64, None, FAKE, None)
    args = lambda **kw: tuple(kw.get(n, v) for n, v in zip(
        ["q", "w", "bias", "L", "B", "T", "Hq", "d", "np", "ns", "logits", "route", "s"], ok))
    assert r(*args(q=None)) == skv.SKV_EINVAL
    assert r(*args(route=None)) == skv.SKV_EINVAL
    assert r(*args(L=0)) == skv.SKV_EINVAL
    assert r(*args(np=0)) == skv.SKV_EINVAL
    assert r(*args(ns=129)) == skv.SKV_EINVAL       # more suffix tokens than tokens
    assert r(*args(q=FAKE + 8)) == skv.SKV_EINVAL   # misaligned
    assert r(*args(w=FAKE + 4)) == skv.SKV_EINVAL
    assert r(*args(Hq=3, d=5)) == skv.SKV_EUNSUPPORTED  # 15 features: not a multiple of 8
    assert r(*args(L=70000)) == skv.SKV_EUNSUPPORTED


def test_select2_rejects_on_host():
    s = skv.lib().attn_select_centroids2
    ok = [FAKE, FAKE, FAKE, FAKE, FAKE, 8, 32, 8, 128, 32, 1024, 4, 102, FAKE, FAKE, FAKE, None]
    def call(**kw):
        names = ["q", "coarse", "co", "fine", "clo", "B", "Hq", "Hkv", "d", "C1", "C", "k1", "k2",
                 "ids", "ss", "se", "s"]
        a = list(ok)
        for k, v in kw.items():
            a[names.index(k)] = v
        return s(*a)
    assert call(q=None) == skv.SKV_EINVAL
    assert call(co=None) == skv.SKV_EINVAL
    assert call(Hq=30) == skv.SKV_EINVAL
    assert call(d=64) == skv.SKV_EUNSUPPORTED
    assert call(k1=0) == skv.SKV_EINVAL
    assert call(k1=33) == skv.SKV_EINVAL        # more coarse clusters kept than exist
    assert call(k2=1025) == skv.SKV_EINVAL
    assert call(C1=2048, k1=4) == skv.SKV_EUNSUPPORTED
    assert call(C=8192) == skv.SKV_EUNSUPPORTED
    assert call(fine=FAKE + 8) == skv.SKV_EINVAL


def test_strerror():
    assert skv.strerror(skv.SKV_OK) == "ok"
    assert "workspace" in skv.strerror(skv.SKV_EWORKSPACE)
    assert skv.strerror(99) == "unknown status"


def test_plan_small_walks_take_the_cluster_schedule():
    # up to 8 tiles per resident CTA (148 SMs x 2 CTAs here) the walk runs as
    # one cluster per KV group and merges in-kernel; one tile more, and the
    # persistent schedule with its record merge takes over
    L = skv.lib()
    small = 148 * 2 * 8  # tiles
    a = good_args(batch=1, q_heads=4, kv_heads=1, max_seq_len=small * 64, max_blocks=small)
    assert L.skv_decode_launches(ctypes.byref(a)) == 1
    assert L.skv_decode_workspace_size(ctypes.byref(a)) == 0
    b = good_args(batch=1, q_heads=4, kv_heads=1, max_seq_len=(small + 1) * 64, max_blocks=small + 1)
    assert L.skv_decode_launches(ctypes.byref(b)) == 2
    assert L.skv_decode_workspace_size(ctypes.byref(b)) > 0


@pytest.mark.parametrize("groups_b,hkv,blocks,want_cb", [
    (16, 8, 512, 16),    # 128 groups of 512 blocks: ~2.3 chunks of a group in flight
    (8, 8, 2048, 32),    # 64 groups of 2048 blocks (a routed stack's full layer)
    (64, 8, 256, 32),    # 512 groups: under one chunk in flight per group
])
def test_plan_art_chunk_length(groups_b, hkv, blocks, want_cb):
    # The ART chunk is 32 blocks when the chunks in flight per group (CTAs /
    # groups) span at most 1/12 of the walk, else 16.  The workspace of a
    # chunk length CB: zeroed control words (item counter, stop chunk per
    # group, ready flag per (group, chunk), consumed and stop per head), per
    # (group, chunk) a look-back record (12 floats) and a partial record (132
    # floats) per head, and per resident CTA (148 SMs x 2) probes of CB blocks
    # x 8 warps x G heads x 12 floats and 8 warps' states of G x 132 floats,
    # both once per post buffer; each of the first two parts rounded up to 256 B.
    L = skv.lib()
    G, NW, ctas = 4, 8, 148 * 2
    src = open(os.path.join(ROOT, "sparse_kv_b200", "csrc", "art.cu")).read()
    posts = int(re.search(r"#define SKV_ART_POSTS (\d+)", src).group(1))
    a = good_args(batch=groups_b, q_heads=hkv * G, kv_heads=hkv, max_seq_len=blocks * 64, max_blocks=blocks,
                  art=_Art(1, 1e-3, 1e-4, 4))
    n = L.skv_decode_workspace_size(ctypes.byref(a))
    groups = groups_b * hkv
    up = lambda x: -(-x // 256) * 256
    sizes = {}
    for cb in (16, 32):
        maxc = -(-blocks // cb)
        items = groups * maxc
        ctl = up((4 + groups + groups * maxc + 2 * groups * G) * 4)
        lb = up(items * G * 12 * 4)
        scratch = ctas * (posts * cb * NW * G * 12 + posts * NW * G * 132) * 4
        sizes[cb] = ctl + lb + scratch + items * G * 132 * 4
    assert n == sizes[want_cb], (n, sizes)


def test_decode_plan_info():
    L = skv.lib()

    def plan(a):
        p = skv.DecodePlan()
        assert L.skv_decode_plan_info(ctypes.byref(a), ctypes.byref(p)) == skv.SKV_OK
        return p

    full = plan(good_args())  # 16 x 8 groups of 512 tiles
    assert (full.schedule, full.ctas, full.splits, full.launches) == (0, 296, 0, 2)
    assert full.workspace_bytes == L.skv_decode_workspace_size(ctypes.byref(good_args()))
    art = plan(good_args(art=_Art(1, 1e-3, 1e-4, 4)))
    assert (art.schedule, art.ctas, art.art_chunk_blocks, art.art_chunks, art.launches) == (2, 296, 16, 32, 2)
    art5 = plan(good_args(batch=8, max_seq_len=131072, max_blocks=2048, art=_Art(1, 1e-3, 1e-4, 4)))
    assert (art5.art_chunk_blocks, art5.art_chunks) == (32, 64)
    small = plan(good_args(batch=1, q_heads=8, kv_heads=2, max_seq_len=4096, max_blocks=64))
    assert (small.schedule, small.splits, small.ctas, small.launches, small.workspace_bytes) == (1, 16, 32, 1, 0)
    seg = plan(good_args(seg_start=FAKE, seg_end=FAKE, n_seg=102))
    assert seg.schedule == 1 and 1 <= seg.splits <= 16 and seg.ctas == seg.splits * 16 * 8
    chunk = plan(good_args(q_tokens=128))
    assert (chunk.schedule, chunk.launches, chunk.workspace_bytes) == (3, 1, 0)
    p = skv.DecodePlan()
    assert L.skv_decode_plan_info(ctypes.byref(good_args(head_dim=64)), ctypes.byref(p)) == skv.SKV_EUNSUPPORTED
    assert L.skv_decode_plan_info(ctypes.byref(good_args()), None) == skv.SKV_EINVAL


def test_decode_plan_from_tensors():
    # the Python binding's view of the plan (host tensors stand in: only their
    # shapes, addresses and alignment are read)
    import torch
    B, Hq, Hkv, L = 1, 8, 2, 4096
    q = torch.zeros((B, 1, Hq, 128), dtype=torch.bfloat16)
    pool = torch.zeros((64, Hkv, 64, 128), dtype=torch.bfloat16)
    bt = torch.zeros((B, 64), dtype=torch.int32)
    sl = torch.full((B,), L, dtype=torch.int32)
    out = torch.zeros((B, 1, Hq, 128), dtype=torch.float32)
    lse = torch.zeros((B, 1, Hq), dtype=torch.float32)
    p = skv.decode_plan(q, pool, pool, bt, sl, out, lse, max_seq_len=L)
    assert p["schedule"] == "cluster" and p["launches"] == 1 and p["workspace_bytes"] == 0
    p = skv.decode_plan(q, pool, pool, bt, sl, out, lse, max_seq_len=L, art=(1e-3, 1e-4, 4))
    assert p["schedule"] == "art" and p["art_chunk_blocks"] in (16, 32)
    with pytest.raises(skv.SkvError):
        skv.decode_plan(q, pool, pool, bt, sl, out, lse, max_seq_len=L, art=(-1.0, 1e-4, 4))


def test_status_of_word_maps_device_bits():
    import sparse_kv_b200 as skv
    B = skv.DEV_BITS
    assert skv.status_of_word(0) == skv.SKV_OK
    assert skv.status_of_word(B["timeout"]) == skv.SKV_ETIMEOUT
    for k in ("bad_page", "bad_seqlen", "bad_order", "bad_segment"):
        assert skv.status_of_word(B[k]) == skv.SKV_EINVAL
    # the binding's bits are the header's SKV_DEV_* values
    import re
    hdr = open(os.path.join(ROOT, "include", "sparsekv.h")).read()
    found = {m.group(1).lower(): int(m.group(2), 16)
             for m in re.finditer(r"#define SKV_DEV_(\w+) (0x[0-9a-fA-F]+)u", hdr)}
    assert found == B
    # a timeout outranks bad-input bits: the outputs are not valid at all
    assert skv.status_of_word(B["timeout"] | B["bad_page"]) == skv.SKV_ETIMEOUT
    assert skv.strerror(skv.SKV_ETIMEOUT) == "device wait timed out"


def test_withhold_hook_validates_and_clears():
    import sparse_kv_b200 as skv
    L = skv.lib()
    assert L.skv_test_withhold_tile(0, -1) == skv.SKV_EINVAL
    assert L.skv_test_withhold_tile(3, 2) == skv.SKV_OK
    assert L.skv_test_withhold_tile(-1, 0) == skv.SKV_OK  # clears the pending hook


def _plan_bytes(B, Hq, Hkv, L, **kw):
    import torch
    import sparse_kv_b200 as skv
    q = torch.zeros(B, 1, Hq, 128, dtype=torch.bfloat16)
    pool = torch.zeros(2, Hkv, 64, 128, dtype=torch.bfloat16)
    bt = torch.zeros(B, (L + 63) // 64, dtype=torch.int32)
    sl = torch.zeros(B, dtype=torch.int32)
    return skv.decode_workspace_size(q, pool, pool, bt, sl, torch.zeros(B, 1, Hq, 128), torch.zeros(B, 1, Hq),
                                     max_seq_len=L, **kw)


def test_static_workspace_holds_the_stated_shapes():
    """The allocation-free entry point's array holds what the header promises
    (148 SMs, as planned without a GPU): ART at the Llama shape for 64 x 32K and
    16 x 128K (the cfg2 and cfg5 ART layers among them) and the persistent
    schedule for 5,500 KV groups at G = 4 (2,800 at G = 8); and refuses a
    larger ART call."""
    import re
    src = open(os.path.join(ROOT, "include", "sparsekv.h")).read()
    m = re.search(r"#define SKV_STATIC_WORKSPACE_BYTES \((\d+)u \* 1024u \* 1024u\)", src)
    cap = int(m.group(1)) * 1024 * 1024
    art = dict(art=(1e-3, 1e-4, 4))
    for B, L in [(16, 32768), (8, 131072), (64, 32768), (16, 131072)]:
        assert 0 < _plan_bytes(B, 32, 8, L, **art) <= cap, (B, L)
    assert _plan_bytes(685, 32, 8, 32768) <= cap        # 5,480 KV groups, no ART
    assert _plan_bytes(345, 64, 8, 32768) <= cap        # 2,760 KV groups at G = 8
    assert _plan_bytes(48, 32, 8, 131072, **art) > cap  # beyond: SKV_EWORKSPACE


def test_binding_argument_counts_match_the_header():
    """Every C function the binding declares takes as many arguments in the
    binding as in include/sparsekv.h (a missing or extra ctypes argument would
    shift every later one)."""
    import re
    src = open(os.path.join(ROOT, "include", "sparsekv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    decls = dict()
    for m in re.finditer(r"SKV_API\s+[\w\s\*]+?\b(\w+)\s*\(([^)]*)\)\s*;", src):
        params = m.group(2).strip()
        decls[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    L = skv.lib()
    checked = 0
    for name, n in decls.items():
        f = getattr(L, name)
        if f.argtypes is not None:
            assert len(f.argtypes) == n, (name, len(f.argtypes), n)
            checked += 1
    assert checked >= 12
