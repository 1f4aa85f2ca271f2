"""A bounded in-kernel wait that runs out, on purpose, on a tiny launch.

calibatt_set_wait_limit shortens the limit of the pipelines' mbarrier waits
of later launches on the device. At 1 ns the first wait that is not already
satisfied (a tile that TMA is still copying) runs out: the kernel records
CALIBATT_ERR_TIMEOUT, winds down without touching further outputs, and drains
the copies and tensor-core work it had issued under the normal limit. The
test checks the status, then restores the limit and checks that the next
launch on the same context is correct against the oracle.

No GPU fault is involved: the waits end by their own limit.
"""
import numpy as np
import pytest
import torch

from calibrated_block_sparse_b200 import synth
from gpu_util import attn_tolerance_ok, bf16_to_f64, energy_bound, require_gpu

pytestmark = pytest.mark.gpu

ERR_TIMEOUT = -6


def _sparse_case(binding, dev):
    q, k, v = synth.plain_qkv(1, 2048, seed=41)
    mask = synth.random_mask(1, 16, 0.5, seed=41)
    rp, ci = _csr(mask)
    work = torch.from_numpy(binding.build_plan(rp, 1, 16)).to(dev)
    return (q, k, v), mask, torch.from_numpy(rp).to(dev), torch.from_numpy(ci).to(dev), work


def _csr(mask):
    h, nb, _ = mask.shape
    rp = np.zeros(h * nb + 1, np.int32)
    rp[1:] = np.cumsum(mask.reshape(h * nb, nb).sum(-1))
    ci = np.nonzero(mask.reshape(h * nb, nb))[1].astype(np.int32)
    return rp, ci


def test_attention_wait_runs_out_then_context_is_usable(oracle):
    binding = require_gpu()
    dev = torch.device("cuda")
    (q, k, v), mask, row_ptr, col_idx, work = _sparse_case(binding, dev)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    assert binding.get_status() == 0
    try:
        binding.set_wait_limit(1e-9)
        binding.sparse_attn_fwd(qd, kd, vd, row_ptr, col_idx, work)
        assert binding.get_status() == ERR_TIMEOUT
    finally:
        binding.set_wait_limit(0.0)
    o, _ = binding.sparse_attn_fwd(qd, kd, vd, row_ptr, col_idx, work)
    assert binding.get_status() == 0
    o_ref, _ = oracle.masked_attention(synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), mask)
    ok, err, bound = attn_tolerance_ok(bf16_to_f64(o), o_ref)
    assert ok, (err, bound)


def test_energy_wait_runs_out_then_context_is_usable(oracle):
    binding = require_gpu()
    dev = torch.device("cuda")
    q, k, _ = synth.plain_qkv(1, 1024, seed=42)
    qd, kd = q.to(dev), k.to(dev)
    for one_pass in (False, True):
        try:
            binding.set_wait_limit(1e-9)
            if one_pass:
                binding.block_energy_1pass(qd, kd, eps=0.9)
            else:
                binding.block_energy(qd, kd, eps=0.9)
            assert binding.get_status() == ERR_TIMEOUT
        finally:
            binding.set_wait_limit(0.0)
    E, _, _, _ = binding.block_energy(qd, kd)
    assert binding.get_status() == 0
    E_ref = oracle.block_energy(synth.bf16_bits(q), synth.bf16_bits(k))
    err = np.abs(E.cpu().numpy().astype(np.float64) - E_ref)
    assert np.all(err <= energy_bound(E_ref))


def test_wait_limit_is_per_device_setting():
    binding = require_gpu()
    lib = binding.load()
    assert lib.calibatt_set_wait_limit(float("nan")) == -1
    assert lib.calibatt_set_wait_limit(120.0) == -1
    assert lib.calibatt_set_wait_limit(0.5) == 0
    assert lib.calibatt_set_wait_limit(0.0) == 0
