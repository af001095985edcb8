"""The C-ABI library loads, exports what include/dsa_indexer.h declares, and
rejects bad arguments on the host before any device work (CPU only)."""
import ctypes
import os
import re

import pytest

import sparse_attention_lightning_tcgen05_b200 as dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa_indexer.h")
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names.update(re.findall(r"\b(dsa_\w+)\s*\(", src))
    return sorted(names)


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 6
    lib = ctypes.CDLL(dsa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(dsa.EXPORTS)


def test_library_does_not_link_libcuda_or_torch():
    # loads on a machine without a driver; cudart is linked statically
    out = os.popen(f"ldd {dsa.LIB_PATH}").read()
    assert "libcuda.so" not in out and "libtorch" not in out and "libc10" not in out


def good_desc(**kw):
    d = dict(T=4, H=64, index_topk=16, S=1024, k_seq_stride=1024 * 128)
    d.update(kw)
    return dsa.make_desc(**d)


def test_workspace_size_on_host():
    assert dsa.dsa_indexer_workspace_size(good_desc()) >= 256


@pytest.mark.parametrize("kw,code", [
    (dict(T=0), dsa.DSA_ERR_INVALID_ARG),
    (dict(H=0), dsa.DSA_ERR_INVALID_ARG),
    (dict(index_topk=0), dsa.DSA_ERR_INVALID_ARG),
    (dict(D=64), dsa.DSA_ERR_UNSUPPORTED),
    (dict(H=300), dsa.DSA_ERR_UNSUPPORTED),
    (dict(S=0), dsa.DSA_ERR_INVALID_ARG),
    (dict(k_seq_stride=1000), dsa.DSA_ERR_INVALID_ARG),
    (dict(k_seq_stride=1023 * 128), dsa.DSA_ERR_INVALID_ARG),
    (dict(mask=dsa.DSA_MASK_CAUSAL, num_seqs=0), dsa.DSA_ERR_INVALID_ARG),
    (dict(dtype=7), dsa.DSA_ERR_INVALID_ARG),
])
def test_bad_descriptors(kw, code):
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_indexer_workspace_size(good_desc(**kw))
    assert e.value.status == code


def compressed_desc(**kw):
    d = dict(T=64, H=64, index_topk=16, S=300, k_seq_stride=0,
             mask=dsa.DSA_MASK_COMPRESSED, compress_ratio=4, query_start=0)
    d.update(kw)
    return dsa.make_desc(**d)


def test_compressed_descriptor_layout():
    """The two compressed-mode fields sit after `mask`, 8-byte aligned, as the
    C header declares them."""
    import ctypes
    f = dsa.dsa_indexer_desc_t
    assert f.query_start.offset % 8 == 0 and f.query_start.offset > f.mask.offset
    assert f.compress_ratio.offset == f.query_start.offset + 8
    assert ctypes.sizeof(f) % 8 == 0
    assert dsa.dsa_indexer_workspace_size(compressed_desc()) >= 256
    assert dsa.dsa_indexer_workspace_size(
        compressed_desc(query_start=2**31 - 1 - 64, compress_ratio=1)) >= 256


@pytest.mark.parametrize("kw,code", [
    (dict(compress_ratio=0), dsa.DSA_ERR_INVALID_ARG),
    (dict(compress_ratio=-4), dsa.DSA_ERR_INVALID_ARG),
    (dict(query_start=-1), dsa.DSA_ERR_INVALID_ARG),
    (dict(S=0), dsa.DSA_ERR_INVALID_ARG),
    (dict(k_seq_stride=300 * 128), dsa.DSA_ERR_INVALID_ARG),   # one pooled cache
    (dict(query_start=1 << 62), dsa.DSA_ERR_UNSUPPORTED),
    (dict(query_start=2**31 - 64), dsa.DSA_ERR_UNSUPPORTED),   # 32-bit positions
    (dict(mask=3), dsa.DSA_ERR_INVALID_ARG),
])
def test_bad_compressed_descriptors(kw, code):
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_indexer_workspace_size(compressed_desc(**kw))
    assert e.value.status == code


def paged_desc(**kw):
    d = dict(T=4, H=64, index_topk=16, S=1000, k_seq_stride=0, page_size=64,
             pages_per_seq=16, num_pages=64, block_table=1 << 20)
    d.update(kw)
    return dsa.make_desc(**d)


def test_paged_descriptor_layout():
    f = dsa.dsa_indexer_desc_t
    assert f.page_size.offset == f.compress_ratio.offset + 4
    assert f.block_table.offset % 8 == 0 and f.block_table.offset == f.num_pages.offset + 4
    assert dsa.dsa_indexer_workspace_size(paged_desc()) >= 256
    assert dsa.dsa_indexer_workspace_size(paged_desc(page_size=16, pages_per_seq=63)) >= 256
    assert dsa.dsa_indexer_workspace_size(paged_desc(dtype=dsa.DSA_KV_FP8_E4M3_E8M0_B32)) >= 256


@pytest.mark.parametrize("kw,code", [
    (dict(page_size=48), dsa.DSA_ERR_INVALID_ARG),            # not a power of two
    (dict(page_size=8, pages_per_seq=125), dsa.DSA_ERR_INVALID_ARG),   # below 16
    (dict(page_size=1 << 17, pages_per_seq=1), dsa.DSA_ERR_INVALID_ARG),
    (dict(pages_per_seq=15), dsa.DSA_ERR_INVALID_ARG),          # S > 15 * 64
    (dict(num_pages=0), dsa.DSA_ERR_INVALID_ARG),
    (dict(k_seq_stride=1000 * 128), dsa.DSA_ERR_INVALID_ARG),   # a pool, not per-token caches
    (dict(mask=dsa.DSA_MASK_CAUSAL, num_seqs=1, cu_seqlens=1 << 20), dsa.DSA_ERR_INVALID_ARG),
    (dict(block_table=(1 << 20) + 2), dsa.DSA_ERR_INVALID_ARG),   # misaligned table
])
def test_bad_paged_descriptors(kw, code):
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_indexer_workspace_size(paged_desc(**kw))
    assert e.value.status == code


def test_compressed_rejects_a_positions_array():
    d = compressed_desc()
    fake = 1 << 20
    for call in (lambda: dsa.dsa_indexer_forward(d, fake, None, fake, fake, None, fake,
                                                 fake, fake, fake, 256),
                 lambda: dsa.dsa_indexer_score(d, fake, None, fake, fake, None, fake,
                                               fake, fake, 256),
                 lambda: dsa.dsa_indexer_topk(d, fake, fake, fake, fake, 256)):
        with pytest.raises(dsa.DsaError) as e:
            call()
        assert e.value.status == dsa.DSA_ERR_INVALID_ARG


def test_bad_pointers_rejected_before_device_work():
    d = good_desc()
    fake = 1 << 20                     # never dereferenced: checks fail first
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_indexer_score(d, None, None, fake, fake, None, fake, fake, fake, 256)
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG
    with pytest.raises(dsa.DsaError) as e:       # misaligned q
        dsa.dsa_indexer_score(d, fake + 2, None, fake, fake, None, fake, fake, fake, 256)
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG
    with pytest.raises(dsa.DsaError) as e:       # positions missing
        dsa.dsa_indexer_forward(d, fake, None, fake, fake, None, None, fake, fake, fake, 256)
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG
    with pytest.raises(dsa.DsaError) as e:       # workspace too small
        dsa.dsa_indexer_forward(d, fake, None, fake, fake, None, fake, fake, fake, fake, 8)
    assert e.value.status == dsa.DSA_ERR_WORKSPACE
    with pytest.raises(dsa.DsaError) as e:       # workspace misaligned
        dsa.dsa_indexer_topk(d, fake, fake, fake, fake + 16, 256)
    assert e.value.status == dsa.DSA_ERR_WORKSPACE
    with pytest.raises(dsa.DsaError) as e:       # no top-k output
        dsa.dsa_indexer_topk(d, fake, fake, None, fake, 256)
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG


def test_status_strings():
    for code in range(7):
        assert dsa.dsa_status_string(code).startswith("DSA_")
    assert dsa.dsa_status_string(99) == "DSA_ERR_UNKNOWN"


def test_valid_call_without_a_gpu_fails_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    fake = 1 << 20
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_indexer_forward(good_desc(), fake, None, fake, fake, None, fake,
                                fake, fake, fake, 256)
    assert e.value.status == dsa.DSA_ERR_CUDA


def test_noalloc_rejects_bad_arguments_on_the_host():
    fake = 1 << 20
    with pytest.raises(dsa.DsaError) as e:       # no top-k output
        dsa.dsa_indexer_forward_noalloc(good_desc(), fake, None, fake, fake, None,
                                        fake, fake, None)
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_indexer_forward_noalloc(good_desc(D=64), fake, None, fake, fake, None,
                                        fake, fake, fake)
    assert e.value.status == dsa.DSA_ERR_UNSUPPORTED


ROW_RULE = os.path.join(os.path.dirname(dsa.LIB_PATH), "csrc", "row_rule.cuh")
_DIV_CHECK = r"""
#include <cstdio>
#include <cstdlib>
#include "row_rule.cuh"
// Every divisor in a list against plain integer division, on numerators
// spread over [0, 2^31) plus the ones next to multiples of the divisor.
int main() {
  const uint32_t ds[] = {1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 16, 17, 31, 32, 33, 64,
                         100, 127, 128, 129, 255, 256, 1000, 4095, 4096, 65535, 65536,
                         65537, 1000003, 16777216, 16777217, 1073741823, 1073741824,
                         1073741825, 2147483646, 2147483647};
  unsigned long long bad = 0, n_checked = 0;
  for (uint32_t d : ds) {
    const dsa::DivMagic g = dsa::div_magic(d);
    auto check = [&](uint64_t n) {
      if (n >= (1ull << 31)) return;
      ++n_checked;
      if (dsa::div_by(static_cast<uint32_t>(n), g) != n / d) ++bad;
    };
    for (uint64_t n = 0; n < 4096; ++n) check(n);
    for (uint64_t n = 0; n < (1ull << 31); n += 65521 + d % 7) check(n);
    for (uint64_t q = 1; q < 4096; ++q) { check(q * d - 1); check(q * d); check(q * d + 1); }
    for (uint64_t n = (1ull << 31) - 4096; n < (1ull << 31); ++n) check(n);
  }
  std::printf("%llu %llu\n", bad, n_checked);
  return bad != 0;
}
"""


def test_invariant_division_of_the_compressed_rule():
    """The kernels' multiply-and-shift division by compress_ratio equals
    integer division for 31-bit numerators (host build of the same header)."""
    import pathlib
    import subprocess
    out_dir = pathlib.Path(__file__).resolve().parent.parent / "_build" / "div_check"
    out_dir.mkdir(parents=True, exist_ok=True)          # _build/ is not versioned
    src = out_dir / "div_check.cpp"
    src.write_text(_DIV_CHECK)
    exe = out_dir / "div_check"
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", os.path.dirname(ROW_RULE), str(src),
                    "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    bad, n = map(int, out.stdout.split())
    assert out.returncode == 0 and bad == 0 and n > 10**6


_LAYOUT = r"""
#include <stddef.h>
#include <stdio.h>
#include "dsa_indexer.h"
#define F(m) printf(#m " %zu\n", offsetof(dsa_indexer_desc_t, m))
int main(void) {
  F(T); F(H); F(D); F(index_topk); F(S); F(k_seq_stride); F(num_seqs);
  F(cu_seqlens); F(dtype); F(mask); F(query_start); F(compress_ratio);
  F(page_size); F(pages_per_seq); F(num_pages); F(block_table); F(flags);
  F(wait_limit_ns); F(cu_seqlens_host);
  printf("sizeof %zu\n", sizeof(dsa_indexer_desc_t));
  return 0;
}
"""


def test_descriptor_layout_matches_the_c_header():
    """Every field of the binding's descriptor sits where a C compiler puts
    it (host build of the header; gcc)."""
    import pathlib
    import subprocess
    out_dir = pathlib.Path(__file__).resolve().parent.parent / "_build" / "layout"
    out_dir.mkdir(parents=True, exist_ok=True)
    src = out_dir / "layout.c"
    src.write_text(_LAYOUT)
    exe = out_dir / "layout"
    subprocess.run(["gcc", "-O0", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    got = dict(line.split() for line in out.strip().splitlines())
    f = dsa.dsa_indexer_desc_t
    for name, off in got.items():
        want = ctypes.sizeof(f) if name == "sizeof" else getattr(f, name).offset
        assert int(off) == want, name


def test_workspace_size_of_a_topk_only_call():
    """With DSA_FLAG_SCORES_IN_WORKSPACE the workspace also holds every score
    row after its 256-byte header: 4*T*S bytes, or 4*sum L_i^2 for packed
    causal rows (from the host copy of cu_seqlens)."""
    import numpy as np
    F = dsa.DSA_FLAG_SCORES_IN_WORKSPACE
    assert dsa.dsa_indexer_workspace_size(good_desc(flags=F)) == 256 + 4 * 4 * 1024
    assert dsa.dsa_indexer_workspace_size(compressed_desc(flags=F)) == 256 + 4 * 64 * 300
    cu = np.array([0, 3, 3, 10, 17], np.int32)
    d = dsa.make_desc(17, 64, 16, mask=dsa.DSA_MASK_CAUSAL, num_seqs=4, cu_seqlens=1 << 20,
                      flags=F, cu_seqlens_host=cu)
    assert dsa.dsa_indexer_workspace_size(d) == 256 + 4 * (9 + 0 + 49 + 49)
    d.flags = 0
    assert dsa.dsa_indexer_workspace_size(d) == 256
    for bad in ([1, 3, 3, 10, 17], [0, 3, 2, 10, 17], [0, 3, 3, 10, 16]):
        arr = np.array(bad, np.int32)
        d = dsa.make_desc(17, 64, 16, mask=dsa.DSA_MASK_CAUSAL, num_seqs=4,
                          cu_seqlens=1 << 20, flags=F, cu_seqlens_host=arr)
        with pytest.raises(dsa.DsaError) as e:
            dsa.dsa_indexer_workspace_size(d)
        assert e.value.status == dsa.DSA_ERR_INVALID_ARG
    d = dsa.make_desc(17, 64, 16, mask=dsa.DSA_MASK_CAUSAL, num_seqs=4, cu_seqlens=1 << 20,
                      flags=F)                       # no host copy to size it from
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_indexer_workspace_size(d)
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG
    with pytest.raises(dsa.DsaError) as e:           # an unknown flag bit
        dsa.dsa_indexer_workspace_size(good_desc(flags=4))
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG


def test_topk_only_forward_host_checks():
    """scores = NULL needs the flag and a workspace that holds the rows;
    both are checked before any device work."""
    fake = 1 << 20
    with pytest.raises(dsa.DsaError) as e:           # no flag
        dsa.dsa_indexer_forward(good_desc(), fake, None, fake, fake, None, fake,
                                None, fake, fake, 1 << 20)
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG
    d = good_desc(flags=dsa.DSA_FLAG_SCORES_IN_WORKSPACE)
    need = dsa.dsa_indexer_workspace_size(d)
    with pytest.raises(dsa.DsaError) as e:           # workspace one float short
        dsa.dsa_indexer_forward(d, fake, None, fake, fake, None, fake,
                                None, fake, fake, need - 4)
    assert e.value.status == dsa.DSA_ERR_WORKSPACE
    with pytest.raises(dsa.DsaError) as e:           # noalloc has no room for rows
        dsa.dsa_indexer_forward_noalloc(d, fake, None, fake, fake, None, fake, None, fake)
    assert e.value.status in (dsa.DSA_ERR_INVALID_ARG, dsa.DSA_ERR_WORKSPACE)



def test_sparse_mqa_host_checks():
    """The sparse-MQA entry points check the descriptor and pointers on the
    host, and size the workspace from the descriptor alone: the header, plus
    the partial results when too few tokens fill the GPU and index rows are
    split into ranges."""
    d = dsa.make_mqa_desc(16, 1, 64, 32768, 2048, 128 ** -0.5)
    n = dsa.dsa_sparse_mqa_workspace_size(d)
    # 16 tokens: each row split into 8 ranges of 256 entries
    assert n == 256 + 16 * 8 * 64 * 130 * 4
    assert dsa.dsa_sparse_mqa_workspace_size(dsa.make_mqa_desc(1, 8192, 64, 8192, 2048, 0.1)) == 256
    for kw, code in ((dict(H=0), dsa.DSA_ERR_INVALID_ARG), (dict(H=129), dsa.DSA_ERR_UNSUPPORTED),
                     (dict(D=64), dsa.DSA_ERR_UNSUPPORTED), (dict(K_top=0), dsa.DSA_ERR_INVALID_ARG),
                     (dict(sm_scale=float("nan")), dsa.DSA_ERR_INVALID_ARG)):
        args = dict(B=2, S=3, H=8, K=100, K_top=64, sm_scale=0.1)
        args.update(kw)
        with pytest.raises(dsa.DsaError) as e:
            dsa.dsa_sparse_mqa_workspace_size(dsa.make_mqa_desc(**args))
        assert e.value.status == code
    fake = 1 << 20
    d = dsa.make_mqa_desc(2, 3, 8, 100, 64, 0.1)
    with pytest.raises(dsa.DsaError) as e:               # misaligned q
        dsa.dsa_sparse_mqa_forward(d, fake + 2, fake, fake, fake, fake, fake, 256)
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG
    with pytest.raises(dsa.DsaError) as e:               # workspace too small
        dsa.dsa_sparse_mqa_forward(d, fake, fake, fake, fake, fake, fake, 128)
    assert e.value.status == dsa.DSA_ERR_WORKSPACE


def test_prepare_host_checks():
    """The front end's descriptor and pointer checks run on the host; its
    workspace is sized from the descriptor alone (the header, plus the fp32
    partial rows of a projection whose K range is split)."""
    d = dsa.make_prepare_desc(16, 64, 7168, 1536, 64)
    n = dsa.dsa_indexer_prepare_workspace_size(d)
    # queries: 64 tiles, 2 splits of 12 K steps -> 2 x 16 x 8192 floats (one
    # wave of 128 items); keys + weights: 1 tile, 28 splits of 4 K steps ->
    # 28 x 16 x 192 floats
    assert n == 256 + max(2 * 16 * 8192 * 4, 28 * 16 * 192 * 4)
    # 300 tokens, K = 256: 3 x 64 query tiles fill the SMs, the key tile
    # splits its 4 K steps in 4
    assert dsa.dsa_indexer_prepare_workspace_size(dsa.make_prepare_desc(300, 64, 256, 256, 64)) == \
        256 + 4 * 300 * 192 * 4
    for kw, code in ((dict(H=24), dsa.DSA_ERR_UNSUPPORTED), (dict(H=144), dsa.DSA_ERR_UNSUPPORTED),
                     (dict(D=64), dsa.DSA_ERR_UNSUPPORTED), (dict(hidden=100), dsa.DSA_ERR_UNSUPPORTED),
                     (dict(rope_dim=63), dsa.DSA_ERR_INVALID_ARG),
                     (dict(rope_dim=130), dsa.DSA_ERR_INVALID_ARG),
                     (dict(k_norm_eps=-1.0), dsa.DSA_ERR_INVALID_ARG),
                     (dict(k_seq_stride=1000), dsa.DSA_ERR_INVALID_ARG)):
        args = dict(T=4, H=64, hidden=256, q_lora_rank=256, rope_dim=64)
        args.update(kw)
        with pytest.raises(dsa.DsaError) as e:
            dsa.dsa_indexer_prepare_workspace_size(dsa.make_prepare_desc(**args))
        assert e.value.status == code
    fake = 1 << 20
    d = dsa.make_prepare_desc(4, 64, 256, 256, 64)
    args = [fake] * 13                                  # x .. key_cache
    args[0] = fake + 2                                   # misaligned x
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_indexer_prepare(d, *args, fake, 256)
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG
    with pytest.raises(dsa.DsaError) as e:               # workspace too small
        dsa.dsa_indexer_prepare(d, *([fake] * 13), fake, 64)
    assert e.value.status == dsa.DSA_ERR_WORKSPACE
