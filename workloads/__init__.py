"""Seeded synthetic workloads shared by the tests, the bench and the oracle runs.

This package draws inputs only: it holds none of GPTQ's arithmetic, so both
the CUDA path and the float64 oracle can be fed from it without sharing code.
"""
from .configs import CONFIGS, Problem, problems_for
from .synth import (cone_activations, gaussian_weights, normal_matrix, spectral_weights,
                    student_t_activations, student_t_weights, swiglu_input)

__all__ = ["CONFIGS", "Problem", "problems_for", "cone_activations",
           "gaussian_weights", "normal_matrix", "spectral_weights",
           "student_t_activations", "student_t_weights", "swiglu_input"]
