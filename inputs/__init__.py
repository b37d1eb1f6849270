"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This package holds shapes, seeds and random draws only: none of the method's
arithmetic lives here.
"""
