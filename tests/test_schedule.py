"""The tensor-core kernels' work decomposition, replayed on the host.

relkl_check_schedule decodes every work item of every part with the helpers
the kernels use and checks that each (unit, row block, column tile) the mask
requires is visited exactly once, that nothing else is, and that every TMA row
coordinate lies inside the tensor.  No GPU is needed, so the schedules of
shapes, masks, padded and packed batches and part splits that the GPU tests
cannot all afford are covered here.
"""
import ctypes
import itertools

import numpy as np
import pytest

from attention_relation_kl_b200 import _abi
from attention_relation_kl_b200._abi import relkl_desc

FAKE = 0x10000   # a non-null device pointer the check never reads


def _desc(B, H, N, d=128, causal=True, lengths=False, n_seq=0, max_seqlen=0):
    x = relkl_desc()
    x.B, x.H, x.N, x.d = B, H, N, d
    x.stride[0], x.stride[1], x.stride[2], x.stride[3] = H * N * d, N * d, d, 1
    x.dtype, x.causal, x.scale, x.reserved = _abi.RELKL_BF16, 1 if causal else 0, 0.0, 0
    x.lengths = FAKE if lengths else None
    if n_seq:
        x.cu_seqlens, x.n_seq, x.max_seqlen = FAKE, n_seq, max_seqlen
    return x


def _check(descs, is_bwd, n_parts, lens=None, cus=None):
    n = len(descs)
    arr = (relkl_desc * n)(*descs)
    keep = []

    def ptrs(lists):
        if lists is None:
            return None
        out = (ctypes.c_void_p * n)()
        for i, v in enumerate(lists):
            if v is not None:
                a = np.ascontiguousarray(v, dtype=np.int32)
                keep.append(a)
                out[i] = a.ctypes.data
        return out

    why = ctypes.create_string_buffer(256)
    code = _abi.lib().relkl_check_schedule(n, arr, is_bwd, n_parts, ptrs(lens), ptrs(cus), why, 256)
    return code, why.value.decode()


@pytest.mark.parametrize("d,causal,is_bwd", list(itertools.product((64, 128), (True, False), (0, 1))))
def test_every_tile_once_for_batched_shapes(d, causal, is_bwd):
    for N in (1, 2, 127, 128, 129, 300, 2049, 4096, 4097, 4480, 8197):
        for n_parts in (1, 2, 3, 7):
            code, why = _check([_desc(2, 3, N, d, causal)], is_bwd, n_parts)
            assert code == 0, (N, n_parts, why)


@pytest.mark.parametrize("causal", [True, False])
def test_fused_relations_with_gqa_heads(causal):
    for is_bwd in (0, 1):
        for N in (300, 4480):
            descs = [_desc(2, 8, N, 128, causal), _desc(2, 2, N, 128, causal),
                     _desc(2, 2, N, 128, causal)]
            assert _check(descs, is_bwd, 1)[0] == 0
            assert _check(descs, is_bwd, 4)[0] == 0


@pytest.mark.parametrize("d", [64, 128])
def test_right_padded_batches(d):
    lens = [[4200, 0, 1, 3001]]
    for causal, is_bwd, n_parts in itertools.product((True, False), (0, 1), (1, 3)):
        code, why = _check([_desc(4, 2, 4200, d, causal, lengths=True)], is_bwd, n_parts, lens=lens)
        assert code == 0, why


@pytest.mark.parametrize("d", [64, 128])
def test_packed_sequences(d):
    seqs = [300, 0, 1, 129, 4300, 57, 4097]
    cu = np.concatenate([[0], np.cumsum(seqs)])
    total = int(cu[-1]) + 11
    for causal, is_bwd, n_parts in itertools.product((True, False), (0, 1), (1, 2, 5)):
        desc = _desc(1, 2, total, d, causal, n_seq=len(seqs), max_seqlen=max(seqs))
        code, why = _check([desc], is_bwd, n_parts, cus=[cu])
        assert code == 0, why
    # short sequences only: the launch sizes its work by max_seqlen
    desc = _desc(1, 1, total, d, True, n_seq=len(seqs), max_seqlen=max(seqs))
    assert _check([desc], 1, 1, cus=[cu])[0] == 0


def test_check_refuses_what_it_cannot_replay():
    # a packed desc without the host offsets, and a CUDA-core shape
    desc = _desc(1, 2, 100, 128, True, n_seq=2, max_seqlen=60)
    assert _check([desc], 0, 1)[0] == _abi.RELKL_ERR_INVALID
    assert _check([_desc(1, 1, 100, 96)], 0, 1)[0] == _abi.RELKL_ERR_UNSUPPORTED
    assert _check([_desc(1, 1, 100, 128)], 0, 0)[0] == _abi.RELKL_ERR_INVALID


def test_backward_kernel_choice_follows_its_cost_rule():
    # relkl_bwd_kernel_for against the rule include/relkl.h states: causal d = 128
    # with 16..32 row blocks takes the paired-block kernel (3) when its rounds of
    # work items, each 1.88 one-block items long, take less than the one-block
    # kernel's (2); fewer row blocks take 2, more take 3
    lib = _abi.lib()

    def choice(descs, sms):
        return lib.relkl_bwd_kernel_for(len(descs), (relkl_desc * len(descs))(*descs), sms)

    for N in (128, 1920, 2048, 2049, 3000, 4096, 4097, 32768):
        nblk = (N + 127) // 128
        for B, H in ((1, 1), (1, 32), (4, 32), (16, 32), (32, 32)):
            for sms in (148, 132, 8):
                one = B * H * ((nblk + 1) // 2)
                pair = B * H * (((nblk + 1) // 2 + 1) // 2)
                if nblk >= 33:
                    want = 3
                elif nblk < 16:
                    want = 2
                else:
                    r1, r2 = -(-one // sms), -(-pair // sms)
                    want = 3 if r2 * 188 < r1 * 100 else 2
                assert choice([_desc(B, H, N)], sms) == want, (N, B, H, sms)
    # the LLaMA2-7B 4K block (Q, K, V of 32 heads: 96 units) keeps the one-block kernel,
    # the sweep's 16 batches of it take the paired one
    qkv = [_desc(1, 32, 4096)] * 3
    assert choice(qkv, 148) == 2 and choice([_desc(16, 32, 4096)] * 3, 148) == 3
    assert choice([_desc(1, 1, 300, causal=False)], 148) == 3       # full mask
    assert choice([_desc(1, 1, 300, d=64)], 148) == 4
    assert choice([_desc(1, 1, 300, d=96)], 148) == 1                # CUDA-core path
    assert choice([_desc(1, 1, 300)], 0) == 0
