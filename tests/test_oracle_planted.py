"""Plant one plausible mistake at a time in a private build of the oracle (on
the CPU) and check that the pins catch it.  The product path is not involved."""
import os
import tempfile

import pytest

import oracle as O
from oracle import build as obuild

import oracle_pins as P

# macro -> the pins expected to catch it
PLANTS = {
    "PLANT_TIE_AWAY": [P.pin_e2m1_rne],
    "PLANT_SR_LE": [P.pin_e2m1_sr],
    "PLANT_SR_NOFLOOR": [P.pin_e2m1_sr],
    "PLANT_MX_NOCLIP_FLOOR": [P.pin_mx_exponent_noclip],
    "PLANT_MX_EMAX": [P.pin_mx_exponent, P.pin_quantize_rne],
    "PLANT_SWIZZLE": [P.pin_swizzle],
    "PLANT_HAD_SIGN_AFTER": [P.pin_hadamard, P.pin_quantize_hadamard],
    "PLANT_NIBBLE_SWAP": [P.pin_packing, P.pin_quantize_rne],
    "PLANT_CTA_TILE_INDEX": [P.pin_gemm_bruteforce],
    "PLANT_GEMM_DROP_TS": [P.pin_gemm_bruteforce, P.pin_gemm_approximates_matmul],
    "PLANT_NV_NO_SENC": [P.pin_nv_scales, P.pin_quantize_rne],
    "PLANT_SWIGLU_SWAP": [P.pin_swiglu],
}


@pytest.fixture(scope="module")
def tmpdir_mod():
    with tempfile.TemporaryDirectory() as d:
        yield d


@pytest.mark.parametrize("macro", sorted(PLANTS))
def test_planted_mistake_is_caught(macro, tmpdir_mod):
    path = obuild.build(out=os.path.join(tmpdir_mod, f"lib_{macro}.so"), defines=(f"-D{macro}",),
                        force=True)
    with O.using(path):
        for pin in PLANTS[macro]:
            with pytest.raises(AssertionError):
                pin()
