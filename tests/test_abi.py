"""The C ABI without a GPU: library loads, exports every declared symbol, struct
layouts agree with a C compiler, the C++ planner matches the oracle planner bit for
bit, and argument errors come back as status codes before any CUDA call."""
import ctypes
import os
import re
import subprocess
import tempfile

import numpy as np
import pytest

import context_blockwise_causal_varlen_b200 as cbv
from oracle import planner as P
from oracle.ring import _block_rows
from synth import cu_from_lengths, packed_doc_lengths, streams

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cbv.h")

pytestmark = pytest.mark.skipif(not os.path.exists(cbv.LIB_PATH), reason="libcbv.so not built")


def test_library_exports_every_declared_symbol():
    names = set(re.findall(r"^(?:int|size_t|const char\*)\s+(cbv_\w+)\s*\(", open(HEADER).read(), re.M))
    assert len(names) >= 20
    L = cbv.lib()
    for n in sorted(names):
        assert hasattr(L, n), n
    assert set(cbv.EXPORTS) == names


def test_struct_layouts_match_the_c_compiler():
    structs = {"cbv_block_fwd_args": cbv.BlockFwdArgs, "cbv_ring_args": cbv.RingArgs,
               "cbv_block_bwd_args": cbv.BlockBwdArgs, "cbv_kvp_args": cbv.KvpArgs, "cbv_decode_args": cbv.DecodeArgs,
               "cbv_cached_ring_args": cbv.CachedRingArgs, "cbv_ring_block": cbv.RingBlock,
               "cbv_row_run": cbv.RowRun, "cbv_ring_step_args": cbv.RingStepArgs, "cbv_diag_args": cbv.DiagArgs}
    src = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HEADER}"', "int main(void){"]
    for cname, st in structs.items():
        src.append(f'printf("{cname} %zu\\n", sizeof({cname}));')
        for f, _ in st._fields_:
            src.append(f'printf("{cname}.{f} %zu\\n", offsetof({cname}, {f}));')
    src.append("return 0;}")
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "l.c")
        exe = os.path.join(d, "l")
        open(c, "w").write("\n".join(src))
        subprocess.run(["gcc", "-o", exe, c], check=True)
        lines = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split("\n")
    got = dict(line.split() for line in lines if line)
    for cname, st in structs.items():
        assert int(got[cname]) == ctypes.sizeof(st), cname
        for f, _ in st._fields_:
            assert int(got[f"{cname}.{f}"]) == getattr(st, f).offset, f"{cname}.{f}"


CUS = [[0, 96, 256], [0, 64], [0, 24, 32, 72], [0, 48, 144, 160], [0, 8, 8, 40]]


@pytest.mark.parametrize("cu", CUS)
@pytest.mark.parametrize("cp", [1, 2, 4])
def test_planner_matches_oracle(cu, cp):
    cu = np.array(cu)
    for layout, name in ((cbv.ZIGZAG, P.ZIGZAG), (cbv.CONTIGUOUS, P.CONTIGUOUS)):
        div = 2 * cp if layout == cbv.ZIGZAG else cp
        if np.any(np.diff(cu) % div):
            with pytest.raises(cbv.CbvError) as e:
                cbv.local_cu_seqlens(cu, cp, layout)
            assert e.value.status == "NOT_DIVISIBLE_2CP"
            continue
        assert np.array_equal(cbv.local_cu_seqlens(cu, cp, layout), P.local_cu_seqlens(cu, cp))
        for r in range(cp):
            assert np.array_equal(cbv.rank_tokens(cu, cp, r, layout), P.rank_tokens(cu, cp, r, name))
        for w in (0, 5, 33):
            assert np.array_equal(cbv.rank_pair_counts(cu, cp, layout, w), P.rank_pair_counts(cu, cp, name, w))
        if layout == cbv.ZIGZAG:
            assert np.array_equal(cbv.half_cu_seqlens(cu, cp), P.half_cu_seqlens(cu, cp))
            cl = P.local_cu_seqlens(cu, cp)
            for front in (True, False):
                assert np.array_equal(cbv.get_half_index(cl, front), P.get_half_index(cl, front))
                lse = np.random.default_rng(0).standard_normal((3, int(cl[-1]))).astype(np.float32)
                assert np.array_equal(cbv.get_half_lse(lse, cl, front), P.get_half_lse(lse, cl, front))
        for r in range(cp):
            for s in range(cp):
                src, kind = cbv.ring_step(r, s, cp, layout)
                osrc, okind = (P.zigzag_step if layout == cbv.ZIGZAG else P.contiguous_step)(r, s, cp)
                names = {0: "diag", 1: "front_k", 2: "back_q", 3: "full", 4: "skip"}
                assert (src, names[kind]) == (osrc, okind)


def test_planner_on_the_packed_workload_and_long_doc():
    for seed in range(5):
        cu = cu_from_lengths(packed_doc_lengths(streams(seed, 6)[4], 16384, 512, 4096, 8))
        for layout, name in ((cbv.ZIGZAG, P.ZIGZAG), (cbv.CONTIGUOUS, P.CONTIGUOUS)):
            assert np.array_equal(cbv.rank_pair_counts(cu, 4, layout), P.rank_pair_counts(cu, 4, name))
        zz = cbv.rank_pair_counts(cu, 4, cbv.ZIGZAG)
        per_doc_equal = True
        for d in range(len(cu) - 1):
            one = cbv.rank_pair_counts(cu[d:d + 2] - cu[d], 4, cbv.ZIGZAG)
            per_doc_equal &= bool(np.all(one == one[0]))
        assert per_doc_equal and np.all(zz == zz[0])
    cu = np.array([0, 65536])
    assert np.all(cbv.rank_pair_counts(cu, 8, cbv.ZIGZAG) == 268439552)
    ct = cbv.rank_pair_counts(cu, 8, cbv.CONTIGUOUS)
    assert ct[0] == 33558528 and ct[-1] == 503320576
    w = cbv.rank_pair_counts(cu, 8, cbv.ZIGZAG, 4096)
    assert w.sum() == 260048896 == P.rank_pair_counts(cu, 8, P.ZIGZAG, 4096).sum()


def _expand(runs, field):
    """The rows of a list of runs, concatenated in order (field: 1 = global row, 4 = local index)."""
    parts = [np.arange(r[field], r[field] + r[2]) for r in runs]
    return np.concatenate(parts).astype(np.int64) if parts else np.zeros(0, np.int64)


def _check_block_descriptors(cu, cp):
    """cbv_plan_zigzag against the oracle's per-(rank, step) blocks, element by element."""
    cu = np.asarray(cu, np.int32)
    for layout, name in ((cbv.ZIGZAG, P.ZIGZAG), (cbv.CONTIGUOUS, P.CONTIGUOUS)):
        div = 2 * cp if layout == cbv.ZIGZAG else cp
        if np.any(np.diff(cu) % div):
            with pytest.raises(cbv.CbvError) as e:
                cbv.plan_zigzag(cu, cp, layout)
            assert e.value.status == "NOT_DIVISIBLE_2CP"
            continue
        blocks = cbv.plan_zigzag(cu, cp, layout)
        want = [(r, s) for r in range(cp) for s in range(cp) if _block_rows(cu, cp, r, s, name) is not None]
        assert [(b["rank"], b["step"]) for b in blocks] == want
        cu_loc, cu_half = P.local_cu_seqlens(cu, cp), P.half_cu_seqlens(cu, cp)
        for b in blocks:
            r, s = b["rank"], b["step"]
            qi, kj, causal, cu_q, cu_k, src = _block_rows(cu, cp, r, s, name)
            assert b["src"] == src and b["causal"] == int(causal)
            # local rows (the flash call's q and k index sets) and their global rows
            assert np.array_equal(_expand(b["q_runs"], 4), qi)
            assert np.array_equal(_expand(b["k_runs"], 4), kj)
            assert np.array_equal(_expand(b["q_runs"], 1), P.rank_tokens(cu, cp, r, name)[qi])
            assert np.array_equal(_expand(b["k_runs"], 1), P.rank_tokens(cu, cp, src, name)[kj])
            # positions are global rows; runs are documents' chunks in local order
            for run in b["q_runs"] + b["k_runs"]:
                d, row0, rows, pos0, _ = run
                assert pos0 == row0 and cu[d] <= row0 and row0 + rows <= cu[d + 1]
            # the cu_seqlens the block's flash call uses on each side
            assert np.array_equal(cu_half if b["q_half"] == 2 else cu_loc, cu_q)
            assert np.array_equal(cu_half if b["k_half"] == 1 else cu_loc, cu_k)
            names = {0: "diag", 1: "front_k", 2: "back_q", 3: "full"}
            step = P.zigzag_step if layout == cbv.ZIGZAG else P.contiguous_step
            assert names[b["kind"]] == step(r, s, cp)[1]


@pytest.mark.parametrize("cu", CUS)
@pytest.mark.parametrize("cp", [1, 2, 4, 8])
def test_block_descriptors_match_the_oracle_blocks(cu, cp):
    _check_block_descriptors(cu, cp)


def test_block_descriptors_of_the_tiny_and_packed_workloads():
    _check_block_descriptors([0, 96, 256], 2)
    for seed in range(3):
        cu = cu_from_lengths(packed_doc_lengths(streams(seed, 6)[4], 16384, 512, 4096, 8))
        _check_block_descriptors(cu, 4)
    _check_block_descriptors([0, 16 * 40, 16 * 41], 8)


def test_block_descriptor_capacity_errors():
    cu = np.array([0, 96, 256], np.int32)
    nb, nr = ctypes.c_int32(0), ctypes.c_int32(0)
    L = cbv.lib()
    assert L.cbv_plan_zigzag(cu.ctypes.data_as(cbv.c_i32p), 2, 2, 0, None, 0, ctypes.byref(nb), None, 0,
                             ctypes.byref(nr)) == 0
    # two documents, two chunks each per rank: the diagonals 4 q + 4 k runs, back-q 2 + 4, front-k 4 + 2
    assert (nb.value, nr.value) == (4, 8 + 6 + 8 + 6)
    blocks = (cbv.RingBlock * nb.value)()
    runs = (cbv.RowRun * (nr.value - 1))()
    rc = L.cbv_plan_zigzag(cu.ctypes.data_as(cbv.c_i32p), 2, 2, 0, blocks, nb.value, ctypes.byref(nb), runs,
                           nr.value - 1, ctypes.byref(nr))
    assert cbv.STATUS[rc] == "BAD_ARG"


def _ring_args(**kw):
    cu = kw.pop("cu", np.array([0, 96, 256], np.int32))
    a = cbv.RingArgs(struct_size=ctypes.sizeof(cbv.RingArgs), abi_version=cbv.ABI_VERSION, total=int(cu[-1]),
                     num_heads=2, num_kv_heads=2, head_dim=64, num_docs=len(cu) - 1,
                     cu_seqlens=cu.ctypes.data_as(cbv.c_i32p), cp=2, causal=1)
    for k, v in kw.items():
        setattr(a, k, v)
    return a, cu


@pytest.mark.parametrize("field,value,status", [
    ("causal", 0, "NOT_CAUSAL"),
    ("head_dim", 96, "UNSUPPORTED_HEAD_DIM"),
    ("num_kv_heads", 3, "GQA_MISMATCH"),
    ("cp", 0, "BAD_ARG"),
    ("cp", 5, "NOT_DIVISIBLE_2CP"),
    ("abi_version", 7, "VERSION"),
    ("struct_size", 8, "VERSION"),
    ("total", 300, "BAD_CU_SEQLENS"),
    ("max_seqlen", 100, "BAD_ARG"),
    ("schedule", 9, "BAD_ARG"),
])
def test_ring_argument_errors_are_reported_before_any_launch(field, value, status):
    a, cu = _ring_args(**{field: value})
    rc = cbv.lib().cbv_zigzag_ring_fwd(ctypes.byref(a), None)
    assert cbv.STATUS[rc] == status, cbv.lib().cbv_last_error_message()
    assert cbv.lib().cbv_last_error_message()
    assert cbv.lib().cbv_zigzag_ring_fwd_workspace_size(ctypes.byref(a)) == 0


def test_bad_cu_seqlens_rejected():
    a, cu = _ring_args(cu=np.array([0, 100, 96, 256], np.int32))
    assert cbv.STATUS[cbv.lib().cbv_zigzag_ring_fwd(ctypes.byref(a), None)] == "BAD_CU_SEQLENS"
    a, cu = _ring_args(cu=np.array([4, 96, 256], np.int32))
    assert cbv.STATUS[cbv.lib().cbv_zigzag_ring_fwd(ctypes.byref(a), None)] == "BAD_CU_SEQLENS"


def test_workspace_sizes_are_reported():
    a, cu = _ring_args()
    n_fwd = cbv.lib().cbv_zigzag_ring_fwd_workspace_size(ctypes.byref(a))
    assert n_fwd >= 256 and n_fwd % 256 == 0
    a.schedule = cbv.SCHEDULE_STEPWISE
    assert cbv.lib().cbv_zigzag_ring_fwd_workspace_size(ctypes.byref(a)) >= 256 * 2 * 64 * 4
    n_bwd = cbv.lib().cbv_zigzag_ring_bwd_workspace_size(ctypes.byref(a))
    assert n_bwd >= 256 * 2 * 64 * 4 + 2 * 256 * 4


def test_decode_rejects_bad_gqa_and_head_dim():
    a = cbv.DecodeArgs(struct_size=ctypes.sizeof(cbv.DecodeArgs), abi_version=cbv.ABI_VERSION, num_seqs=1, total_q=1,
                       total_k=1, num_heads=32, num_kv_heads=1, head_dim=128)
    assert cbv.STATUS[cbv.lib().cbv_varlen_decode(ctypes.byref(a), None)] == "GQA_MISMATCH"
    a.num_kv_heads, a.num_heads = 4, 30
    assert cbv.STATUS[cbv.lib().cbv_varlen_decode(ctypes.byref(a), None)] == "GQA_MISMATCH"
    a.num_heads, a.head_dim = 32, 80
    assert cbv.STATUS[cbv.lib().cbv_varlen_decode(ctypes.byref(a), None)] == "UNSUPPORTED_HEAD_DIM"


def test_kvp_rejects_bad_block_and_segment_sizes():
    a = cbv.KvpArgs(struct_size=ctypes.sizeof(cbv.KvpArgs), abi_version=cbv.ABI_VERSION, q_len=16, num_heads=4,
                    num_kv_heads=2, head_dim=128, num_blocks=8, block_size=24, shards=2, blocks_per_shard=4,
                    seg_size=512)
    assert cbv.STATUS[cbv.lib().cbv_kvp_segmented_prefill(ctypes.byref(a), None)] == "BAD_ARG"
    a.block_size, a.seg_size = 32, 0
    assert cbv.STATUS[cbv.lib().cbv_kvp_segmented_prefill(ctypes.byref(a), None)] == "BAD_ARG"
    a.block_size, a.seg_size = 4, 512
    assert cbv.STATUS[cbv.lib().cbv_kvp_segmented_prefill(ctypes.byref(a), None)] == "BAD_ARG"


def test_empty_problems_return_ok_without_touching_the_device():
    # no rows: every entry point validates its arguments and returns before any CUDA call
    for cu in (np.array([0], np.int32), np.array([0, 0, 0], np.int32)):
        a, _ = _ring_args(cu=cu)
        assert cbv.lib().cbv_zigzag_ring_fwd(ctypes.byref(a), None) == 0, cbv.lib().cbv_last_error_message()
        assert cbv.lib().cbv_zigzag_ring_bwd(ctypes.byref(a), None) == 0, cbv.lib().cbv_last_error_message()
    assert cbv.lib().cbv_attn_merge(None, None, None, cbv.DTYPE_F32, None, None, 0, 2, 128, None) == 0
    d = cbv.DecodeArgs(struct_size=ctypes.sizeof(cbv.DecodeArgs), abi_version=cbv.ABI_VERSION, num_seqs=0, total_q=0,
                       total_k=0, num_heads=8, num_kv_heads=2, head_dim=128)
    assert cbv.lib().cbv_varlen_decode(ctypes.byref(d), None) == 0
    # but a malformed empty call is still an error
    a, _ = _ring_args(cu=np.array([0], np.int32), head_dim=80)
    assert cbv.STATUS[cbv.lib().cbv_zigzag_ring_fwd(ctypes.byref(a), None)] == "UNSUPPORTED_HEAD_DIM"


def _cached_args(**kw):
    cu = kw.pop("cu", np.array([0, 96, 256], np.int32))
    a = cbv.CachedRingArgs(struct_size=ctypes.sizeof(cbv.CachedRingArgs), abi_version=cbv.ABI_VERSION, num_blocks=3,
                           total=int(cu[-1]), num_heads=4, num_kv_heads=2, head_dim=128, num_docs=len(cu) - 1,
                           cu_seqlens=cu.ctypes.data_as(cbv.c_i32p), cp=2)
    for k, v in kw.items():
        setattr(a, k, v)
    return a, cu


@pytest.mark.parametrize("field,value,status", [
    ("num_blocks", 0, "BAD_ARG"),
    ("num_blocks", 9, "BAD_ARG"),
    ("head_dim", 96, "UNSUPPORTED_HEAD_DIM"),
    ("num_kv_heads", 3, "GQA_MISMATCH"),
    ("cp", 5, "NOT_DIVISIBLE_2CP"),
    ("struct_size", 8, "VERSION"),
    ("layout", 4, "BAD_ARG"),
])
def test_cached_ring_argument_errors_are_reported_before_any_launch(field, value, status):
    a, cu = _cached_args(**{field: value})
    for f in (cbv.lib().cbv_cached_ring_fwd, cbv.lib().cbv_cached_ring_bwd):
        assert cbv.STATUS[f(ctypes.byref(a), None)] == status, cbv.lib().cbv_last_error_message()
    assert cbv.lib().cbv_cached_ring_fwd_workspace_size(ctypes.byref(a)) == 0
    assert cbv.lib().cbv_cached_ring_bwd_workspace_size(ctypes.byref(a)) == 0


def test_cached_ring_workspace_holds_the_fp32_block_output():
    a, cu = _cached_args()
    n = cbv.lib().cbv_cached_ring_fwd_workspace_size(ctypes.byref(a))
    assert n >= 256 * 4 * 128 * 4  # block 0's normalised output in fp32
    a.num_blocks = 1  # the sequence alone: the plain ring forward's scratch
    r, _ = _ring_args(num_heads=4, head_dim=128)
    assert cbv.lib().cbv_cached_ring_fwd_workspace_size(ctypes.byref(a)) == \
        cbv.lib().cbv_zigzag_ring_fwd_workspace_size(ctypes.byref(r))
    assert cbv.lib().cbv_cached_ring_bwd_workspace_size(ctypes.byref(a)) == \
        cbv.lib().cbv_zigzag_ring_bwd_workspace_size(ctypes.byref(r))
    a, _ = _cached_args(cu=np.array([0, 0], np.int32))
    assert cbv.lib().cbv_cached_ring_fwd(ctypes.byref(a), None) == 0
    assert cbv.lib().cbv_cached_ring_bwd(ctypes.byref(a), None) == 0


def test_argument_errors_launch_nothing():
    n0 = cbv.launch_count()
    a, _ = _ring_args(head_dim=96)
    assert cbv.STATUS[cbv.lib().cbv_zigzag_ring_fwd(ctypes.byref(a), None)] == "UNSUPPORTED_HEAD_DIM"
    a, _ = _ring_args(cu=np.array([0], np.int32))
    assert cbv.lib().cbv_zigzag_ring_bwd(ctypes.byref(a), None) == 0
    assert cbv.launch_count() == n0


def _block_args(**kw):
    cq = np.array([0, 64, 160], np.int32)
    ck = np.array([0, 96, 200], np.int32)
    a = cbv.BlockFwdArgs(struct_size=ctypes.sizeof(cbv.BlockFwdArgs), abi_version=cbv.ABI_VERSION, q=256, k=512,
                         v=768, total_q=160, total_k=200, num_heads=4, num_kv_heads=2, head_dim=128, num_docs=2,
                         cu_seqlens_q=cq.ctypes.data_as(cbv.c_i32p), cu_seqlens_k=ck.ctypes.data_as(cbv.c_i32p),
                         causal=1, out_dtype=cbv.DTYPE_BF16, out=1024, lse=2048)
    for k, v in kw.items():
        setattr(a, k, v)
    return a, (cq, ck)


@pytest.mark.parametrize("field,value,status", [
    ("merge", 1, "BAD_DTYPE"),       # merging needs the f32 running out
    ("out_dtype", 7, "BAD_DTYPE"),
    ("q", 8, "MISALIGNED"),
    ("out", 1032, "MISALIGNED"),
    ("workspace", None, "WORKSPACE_TOO_SMALL"),
])
def test_block_forward_argument_errors(field, value, status):
    # fake device addresses: every one of these is refused on the host, before any CUDA call
    a, keep = _block_args(**{field: value})
    rc = cbv.lib().cbv_attn_block_fwd(ctypes.byref(a), None)
    assert cbv.STATUS[rc] == status, cbv.lib().cbv_last_error_message()


def _kvp_args(**kw):
    a = cbv.KvpArgs(struct_size=ctypes.sizeof(cbv.KvpArgs), abi_version=cbv.ABI_VERSION, q=256, q_stride_head=16 * 128,
                    q_stride_token=128, q_len=16, num_heads=4, num_kv_heads=2, head_dim=128, k_cache=512, v_cache=768,
                    num_blocks=8, block_size=32, shards=2, blocks_per_shard=4, kv_mode=cbv.KV_ROUND_ROBIN,
                    seg_size=128, global_q_offset=100, out=1024)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("field,value,status", [
    ("kv_mode", 5, "BAD_ARG"),
    ("global_q_offset", -1, "BAD_ARG"),
    ("shard_out", 4096, "BAD_ARG"),   # per-shard out without per-shard lse
    ("q", 8, "MISALIGNED"),
    ("q_stride_token", 132, "MISALIGNED"),
    ("shards", 0, "BAD_SHAPE"),
    ("num_kv_heads", 3, "GQA_MISMATCH"),
    ("workspace", None, "WORKSPACE_TOO_SMALL"),
    ("shard_base", -1, "BAD_ARG"),
    ("total_shards", 1, "BAD_ARG"),   # the call's two shards do not fit in one
    ("shard_base", 1, "BAD_ARG"),     # shards 1 and 2 of two (total_shards 0: the call's own count)
])
def test_prefill_argument_errors(field, value, status):
    a = _kvp_args(**{field: value})
    rc = cbv.lib().cbv_kvp_segmented_prefill(ctypes.byref(a), None)
    assert cbv.STATUS[rc] == status, cbv.lib().cbv_last_error_message()


def test_prefill_shard_range_within_the_total():
    # shards 2 and 3 of four pass the checks (the call then stops at the missing workspace); 3 and 4 do not
    ok = _kvp_args(shard_base=2, total_shards=4)
    assert cbv.STATUS[cbv.lib().cbv_kvp_segmented_prefill(ctypes.byref(ok), None)] == "WORKSPACE_TOO_SMALL"
    assert cbv.lib().cbv_kvp_workspace_size(ctypes.byref(ok)) > 0
    bad = _kvp_args(shard_base=3, total_shards=4)
    assert cbv.STATUS[cbv.lib().cbv_kvp_segmented_prefill(ctypes.byref(bad), None)] == "BAD_ARG"
    assert cbv.lib().cbv_kvp_workspace_size(ctypes.byref(bad)) == 0


@pytest.mark.parametrize("field,value,status", [
    ("dout", None, "BAD_ARG"),
    ("dq_acc", 4104, "MISALIGNED"),
    ("head_dim", 256, "UNSUPPORTED_HEAD_DIM"),
    ("total_k", 150, "BAD_CU_SEQLENS"),   # the key offsets run past the key rows
    ("workspace", None, "WORKSPACE_TOO_SMALL"),
])
def test_block_backward_argument_errors(field, value, status):
    cq = np.array([0, 64, 160], np.int32)
    ck = np.array([0, 96, 200], np.int32)
    a = cbv.BlockBwdArgs(struct_size=ctypes.sizeof(cbv.BlockBwdArgs), abi_version=cbv.ABI_VERSION, dout=256, q=512,
                         k=768, v=1024, out=1280, lse=1536, total_q=160, total_k=200, num_heads=4, num_kv_heads=2,
                         head_dim=128, num_docs=2, cu_seqlens_q=cq.ctypes.data_as(cbv.c_i32p),
                         cu_seqlens_k=ck.ctypes.data_as(cbv.c_i32p), causal=1, dq_acc=2048, dk_acc=2304, dv_acc=2560)
    setattr(a, field, value)
    rc = cbv.lib().cbv_attn_block_bwd(ctypes.byref(a), None)
    assert cbv.STATUS[rc] == status, cbv.lib().cbv_last_error_message()


def test_stalled_forward_diagnostic_checks_its_limit_before_any_launch():
    a, cu = _ring_args()
    L = cbv.lib()
    n0 = cbv.launch_count()
    for lim in (0, 99_999, 2_000_000_000):
        assert cbv.STATUS[L.cbv_debug_ring_fwd_stalled(ctypes.byref(a), lim, None)] == "BAD_ARG"
    a.schedule = cbv.SCHEDULE_STEPWISE
    assert cbv.STATUS[L.cbv_debug_ring_fwd_stalled(ctypes.byref(a), 1_000_000, None)] == "BAD_ARG"
    assert cbv.launch_count() == n0


def _step_args(**kw):
    cu = kw.pop("cu", np.array([0, 96, 256], np.int32))
    a = cbv.RingStepArgs(struct_size=ctypes.sizeof(cbv.RingStepArgs), abi_version=cbv.ABI_VERSION, rank=0, step=0,
                         n_local=int(cu[-1]) // 2, num_heads=2, num_kv_heads=2, head_dim=64, num_docs=len(cu) - 1,
                         cu_seqlens=cu.ctypes.data_as(cbv.c_i32p), cp=2)
    for k, v in kw.items():
        setattr(a, k, v)
    return a, cu


@pytest.mark.parametrize("field,value,status", [
    ("rank", 2, "BAD_ARG"), ("step", -1, "BAD_ARG"), ("cp", 0, "BAD_ARG"), ("n_local", 100, "BAD_CU_SEQLENS"),
    ("head_dim", 96, "UNSUPPORTED_HEAD_DIM"), ("num_kv_heads", 3, "GQA_MISMATCH"), ("abi_version", 3, "VERSION"),
    ("layout", 5, "BAD_ARG"),
])
def test_ring_step_argument_errors_are_reported_before_any_launch(field, value, status):
    a, cu = _step_args(**{field: value})
    L = cbv.lib()
    n0 = cbv.launch_count()
    for fn in (L.cbv_ring_step_fwd, L.cbv_ring_step_bwd):
        assert cbv.STATUS[fn(ctypes.byref(a), None)] == status
    assert L.cbv_ring_step_fwd_workspace_size(ctypes.byref(a)) == 0
    assert cbv.launch_count() == n0


def test_ring_step_workspace_sizes_are_reported():
    a, cu = _step_args()
    L = cbv.lib()
    assert L.cbv_ring_step_fwd_workspace_size(ctypes.byref(a)) > 256
    assert L.cbv_ring_step_bwd_workspace_size(ctypes.byref(a)) > 256


def test_diag_and_layout_helper_errors():
    L = cbv.lib()
    a = cbv.DiagArgs(struct_size=ctypes.sizeof(cbv.DiagArgs), abi_version=cbv.ABI_VERSION, num_blocks=9, total=4,
                     num_heads=2, num_kv_heads=2, head_dim=64)
    assert cbv.STATUS[L.cbv_cached_diag_merge(ctypes.byref(a), None)] == "BAD_ARG"
    a.num_blocks, a.head_dim = 2, 80
    assert cbv.STATUS[L.cbv_cached_diag_grad(ctypes.byref(a), None)] == "UNSUPPORTED_HEAD_DIM"
    assert cbv.STATUS[L.cbv_convert_f32_bf16(None, None, 6, 1.0, None)] == "BAD_SHAPE"
    assert cbv.STATUS[L.cbv_swap_leading_axes(None, None, 2, 2, 6, None)] == "BAD_SHAPE"
    assert L.cbv_swap_leading_axes(None, None, 0, 2, 8, None) == 0  # nothing to move


@pytest.mark.parametrize("seed", range(12))
def test_block_descriptors_on_random_document_mixes(seed):
    # random document counts and lengths (multiples of 2 cp, empty documents included) for every cp
    rng = np.random.default_rng(500 + seed)
    cp = int(rng.choice([1, 2, 3, 4, 8]))
    n = int(rng.integers(1, 9))
    lengths = rng.integers(0, 12, n) * 2 * cp
    _check_block_descriptors(cu_from_lengths(lengths), cp)

