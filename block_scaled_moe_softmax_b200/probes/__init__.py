"""Measurement probes behind design choices of the library (not part of the layer)."""
